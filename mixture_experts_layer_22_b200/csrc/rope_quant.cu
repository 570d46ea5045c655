// rope_quant.cu - inverse rotary embedding fused with per-head E4M3
// quantisation, the attention-side kernel the Russian summary names in its
// section "Убрать лишние JIT-перекомпиляции Triton": rotary embedding and FP8
// quantisation in one pass, with the token count a run-time argument (a
// recompile per num_tokens cost 9% of time-to-first-token there).  Here the
// token count is a kernel argument like any other; nothing is specialised on
// it.
//
// For each token t (position p = positions[t]) and head h, the head vector y
// (bf16) is rotated back by the angle of its position: each pair (a', b'),
// (i, i + rot_dim/2) or (2i, 2i + 1), becomes
//     a = a' c + b' s,   b = b' c - a' s,   c = cos_sin[p][i], s = cos_sin[p][rot_dim/2 + i],
// elements beyond rot_dim pass through; then the head's scale is
// amax(|r|) / 448 (1 when r is all zero) and each element's code is
// E4M3(r / scale), round to nearest even, saturated.  The arithmetic is fp32
// with every product and sum rounded on its own (no fused multiply-add) and
// IEEE division, so a code is decided the same way wherever it is computed.
//
// Layout: head_dim / 8 lanes per head, 8 consecutive elements per lane (one
// 16-byte load), several heads per warp; see the kernel.  HBM-bound once the
// per-element arithmetic is lean: per head 2*head_dim bytes in, head_dim + 4
// bytes out.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "common.cuh"

namespace moe {

// The quotient r / scale, correctly rounded, from the correctly rounded
// reciprocal rs = RN(1 / scale) of the head: q = RN(r rs) is within an ulp of
// r / scale, the residual r - q scale is exact in one fused multiply-add, and
// RN(q + residual rs) is then the correctly rounded quotient (Markstein's
// theorem on division by reciprocal refinement, "IA-64 and Elementary
// Functions", 2000).  The residual is a multiple of about 2^(e_r - 46), so it
// is exact (if need be as a subnormal) for |r| >= 2^-103.  With
// 2^-60 <= amax <= 2^100 the scale and rs are normal, and an element can only
// get a nonzero code when |r| >= amax 2^-19 >= 2^-79, well inside that range;
// smaller elements get a quotient below 2^-10 of the right sign, hence the same
// code (+-0) as the exact quotient.  For amax outside the range the IEEE
// division is used.
__device__ __forceinline__ float div_by_scale(float r, float scale, float rs)
{
    const float q = __fmul_rn(r, rs);
    const float res = __fmaf_rn(-q, scale, r);
    return __fmaf_rn(res, rs, q);
}

// Eight bf16 values (one 16-byte load) to fp32.
__device__ __forceinline__ void load8_bf16(const void *p, float (&y)[8])
{
    const uint4 v = __ldg(reinterpret_cast<const uint4 *>(p));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        y[2 * i] = __uint_as_float(w[i] << 16);
        y[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

// Each head is handled by kL = head_dim / 8 lanes, 8 consecutive elements
// per lane (one 16-byte load), so a warp processes 32 / kL heads at once and
// shares the per-head reduction and scale arithmetic among them.  A warp
// takes one token and a chunk of hc of its heads: the token's position and
// the rotary coefficients of the lane's 8 elements are loaded once for the
// chunk.  Pair partners: the neighbouring element of the same lane
// (interleaved pairs) or the same element of the lane kL/2 ... away
// (neox pairs, rot_dim a multiple of 16: a shuffle).
template <int kL, bool kInterleaved>
__global__ void __launch_bounds__(256, 3) inv_rope_quant_kernel(const __nv_bfloat16 *__restrict__ x,
                                                             const int32_t *__restrict__ positions,
                                                             const float *__restrict__ cos_sin, int T, int n_heads,
                                                             int rot_dim, int max_pos, int hc, uint8_t *q,
                                                             float *scales, int32_t *status)
{
    constexpr int kHd = 8 * kL;
    constexpr int kHpw = 32 / kL;                  // heads per warp pass
    const int lane = threadIdx.x & 31;
    const int warp_g = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int n_warps = (gridDim.x * blockDim.x) >> 5;
    const int sub = lane / kL, li = lane % kL;     // head within the pass, lane within the head
    const int half = rot_dim >> 1;
    const int n_chunks = (n_heads + hc - 1) / hc;
    const long long n_items = static_cast<long long>(T) * n_chunks;
    // this lane's elements j = 8 li + v: rotated or not, first of its pair,
    // pair index; neox partners sit half / 8 lanes away in the same register.
    // A lane's 8 elements are all rotated, all passed through, or (a partial
    // rotary width that is not a multiple of 8) mixed.
    const int pl = half >> 3;
    const bool all_rot = 8 * li + 8 <= rot_dim, none_rot = 8 * li >= rot_dim;
    bool rotated[8], first[8];
    int pidx[8];
#pragma unroll
    for (int v = 0; v < 8; ++v) {
        const int j = 8 * li + v;
        rotated[v] = j < rot_dim;
        if (kInterleaved) {
            first[v] = (v & 1) == 0;
            pidx[v] = j >> 1;
        } else {
            first[v] = j < half;
            pidx[v] = first[v] ? j : j - half;
        }
    }
    for (long long item = warp_g; item < n_items; item += n_warps) {
        const int t = static_cast<int>(item / n_chunks);
        const int h_begin = static_cast<int>(item % n_chunks) * hc;
        const int h_end = min(n_heads, h_begin + hc);
        const int p = __ldg(positions + t);
        const long long row = static_cast<long long>(t) * n_heads;
        if (p < 0 || p >= max_pos) {                    // the same for the whole warp
            if (lane == 0 && status) set_status(status, MOE_ERR_DEVICE_CHECK);
            for (int h = h_begin + sub; h < h_end; h += kHpw) {
                if (li == 0) scales[row + h] = 0.0f;
                *reinterpret_cast<uint2 *>(q + (row + h) * kHd + 8 * li) = make_uint2(0u, 0u);
            }
            continue;
        }
        // cos and the sine signed for the element's place in its pair:
        // a = a' c + b' s, b = b' c + a' (-s), each term rounded, so the same
        // bits as the difference b' c - a' s
        const float *cs = cos_sin + static_cast<size_t>(p) * rot_dim;
        float c[8], sn[8];
#pragma unroll
        for (int v = 0; v < 8; ++v) {
            c[v] = rotated[v] ? __ldg(cs + pidx[v]) : 0.0f;
            const float sv = rotated[v] ? __ldg(cs + half + pidx[v]) : 0.0f;
            sn[v] = first[v] ? sv : -sv;
        }
        // kP passes of kHpw heads at a time: every load of the kP passes is
        // issued before any is used (more bytes in flight per lane)
        constexpr int kP = 4;
        for (int h00 = h_begin; h00 < h_end; h00 += kP * kHpw) {
            float y[kP][8];
#pragma unroll
            for (int u = 0; u < kP; ++u) {
                const int h = h00 + u * kHpw + sub;
                if (h < h_end) load8_bf16(x + (row + h) * kHd + 8 * li, y[u]);
                else
#pragma unroll
                    for (int v = 0; v < 8; ++v) y[u][v] = 0.0f;
            }
#pragma unroll
            for (int u = 0; u < kP; ++u) {
                const int h = h00 + u * kHpw + sub;
                if (h00 + u * kHpw >= h_end) break;        // uniform across the warp
                float yp[8], r[8];
#pragma unroll
                for (int v = 0; v < 8; ++v)
                    yp[v] = kInterleaved ? y[u][v ^ 1] : __shfl_xor_sync(0xffffffffu, y[u][v], pl);
                if (all_rot) {
#pragma unroll
                    for (int v = 0; v < 8; ++v) r[v] = __fadd_rn(__fmul_rn(y[u][v], c[v]), __fmul_rn(yp[v], sn[v]));
                } else if (none_rot) {
#pragma unroll
                    for (int v = 0; v < 8; ++v) r[v] = y[u][v];
                } else {
#pragma unroll
                    for (int v = 0; v < 8; ++v)
                        r[v] = rotated[v] ? __fadd_rn(__fmul_rn(y[u][v], c[v]), __fmul_rn(yp[v], sn[v])) : y[u][v];
                }
                float amax = 0.0f;
#pragma unroll
                for (int v = 0; v < 8; ++v) amax = fmaxf(amax, fabsf(r[v]));
#pragma unroll
                for (int o = kL / 2; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
                const float sc = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
                const float rs = __frcp_rn(sc);
                float qv[8];
                if (amax >= 0x1p-60f && amax <= 0x1p100f) {
#pragma unroll
                    for (int v = 0; v < 8; ++v) qv[v] = div_by_scale(r[v], sc, rs);
                } else {
#pragma unroll
                    for (int v = 0; v < 8; ++v) qv[v] = __fdiv_rn(r[v], sc);
                }
                uint32_t w[2] = {0u, 0u};
#pragma unroll
                for (int v = 0; v < 8; v += 2) {
                    const float2 qq = make_float2(qv[v], qv[v + 1]);
                    const uint32_t pair =
                        static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(qq, __NV_SATFINITE, __NV_E4M3)) & 0xFFFFu;
                    w[v >> 2] |= pair << ((v & 2) * 8);
                }
                if (h < h_end) {
                    *reinterpret_cast<uint2 *>(q + (row + h) * kHd + 8 * li) = make_uint2(w[0], w[1]);
                    if (li == 0) scales[row + h] = sc;
                }
            }
        }
    }
}

}  // namespace moe

using namespace moe;

extern "C" int moe_inv_rope_quant_per_head(const moe_rope_shape_t *shape, const void *x, const int32_t *positions,
                                           const float *cos_sin, uint8_t *q, float *scales, int32_t *status,
                                           moe_stream_t stream)
{
    int &launches = launch_counter();
    launches = 0;
    if (!shape) return MOE_ERR_INVALID_ARG;
    const moe_rope_shape_t &s = *shape;
    if (s.num_tokens < 0 || s.n_heads < 1 || s.max_pos < 1 || s.rot_dim < 2 || (s.rot_dim & 1) ||
        s.rot_dim > s.head_dim || (s.interleaved != 0 && s.interleaved != 1))
        return MOE_ERR_INVALID_ARG;
    if (s.head_dim != 64 && s.head_dim != 128 && s.head_dim != 256) return MOE_ERR_UNSUPPORTED;
    if (!s.interleaved && s.rot_dim % 16 != 0) return MOE_ERR_UNSUPPORTED;
    if (static_cast<int64_t>(s.num_tokens) * s.n_heads > (int64_t(1) << 40)) return MOE_ERR_INVALID_ARG;
    if (s.num_tokens == 0) return MOE_OK;
    if (!x || !positions || !cos_sin || !q || !scales) return MOE_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(q) & 7) ||
        (reinterpret_cast<uintptr_t>(cos_sin) & 3) || (reinterpret_cast<uintptr_t>(scales) & 3))
        return MOE_ERR_INVALID_ARG;
    // heads per warp item: all of a token's heads when there are enough tokens
    // to give every SM 32 warps, else fewer so that small batches still spread
    // over the GPU
    const int hpw = 32 / (s.head_dim / 8);
    int hc = s.n_heads;
    while (hc > hpw && static_cast<long long>(s.num_tokens) * ((s.n_heads + hc - 1) / hc) < 148LL * 32)
        hc = ((hc / 2) + hpw - 1) / hpw * hpw;
    const long long items = static_cast<long long>(s.num_tokens) * ((s.n_heads + hc - 1) / hc);
    const long long want = (items + 7) / 8;
    const int blocks = static_cast<int>(want < 148 * 8 ? want : 148 * 8);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const __nv_bfloat16 *xb = static_cast<const __nv_bfloat16 *>(x);
#define MOE_ROPE(L, IL)                                                                                      \
    inv_rope_quant_kernel<L, IL><<<blocks, 256, 0, st>>>(xb, positions, cos_sin, s.num_tokens, s.n_heads,    \
                                                          s.rot_dim, s.max_pos, hc, q, scales, status)
    const int L = s.head_dim / 8;
    if (s.interleaved) {
        if (L == 8) MOE_ROPE(8, true);
        else if (L == 16) MOE_ROPE(16, true);
        else MOE_ROPE(32, true);
    } else {
        if (L == 8) MOE_ROPE(8, false);
        else if (L == 16) MOE_ROPE(16, false);
        else MOE_ROPE(32, false);
    }
#undef MOE_ROPE
    launches = 1;
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
