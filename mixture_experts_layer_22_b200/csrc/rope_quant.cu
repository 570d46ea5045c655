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
// Layout: head_dim / 16 lanes per head, 16 elements per lane in two 16-byte
// loads chosen so that both elements of every rotary pair sit in the lane,
// several heads per warp; see the kernel.  HBM-bound once the per-element
// arithmetic is lean: per head 2*head_dim bytes in, head_dim + 4 bytes out.
#include <atomic>

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
// smaller elements get a quotient below 2^-10, hence the code +-0 of the
// exact quotient, once the sign is right.  The sign needs one fix: for
// r = -0, q is -0 and the residual +0, and their sum rounds to +0.  The
// quotient of r by a positive scale has r's sign, so it is taken from r
// (with_sign_of).  For amax outside the range the IEEE division is used.
__device__ __forceinline__ float with_sign_of(float q, float r)
{
    return __int_as_float((__float_as_int(q) & 0x7FFFFFFF) | (__float_as_int(r) & static_cast<int>(0x80000000u)));
}

// amax / 448 correctly rounded, for normal results: 448 = 7 * 64, and a
// division by 64 is exact, so RN(amax / 448) = RN(amax / 7) * 2^-6; the
// division by 7 is the same reciprocal refinement with RN(1/7).
__device__ __forceinline__ float div448(float amax)
{
    constexpr float kRcp7 = 0.142857149f;       // RN(1/7)
    const float q = __fmul_rn(amax, kRcp7);
    const float res = __fmaf_rn(-q, 7.0f, amax);
    return __fmul_rn(__fmaf_rn(res, kRcp7, q), 0x1p-6f);
}

// A pair of fp32 lanes: the packed fp32x2 multiply, add and fused
// multiply-add of sm_100 take one instruction for two elements, each element
// rounded exactly like the scalar operation.  The compiler, however, fuses a
// packed product whose only use is a packed sum into one packed fused
// multiply-add, explicit rounding modes and --fmad=false notwithstanding
// (measured: a 1-ulp change in about one head in six).  sum2 therefore forms
// the separately rounded sum p + q as fma(q, one, p) with `one` a run-time
// 1.0 the compiler cannot see through: q * one is exact, so the result is
// RN(p + q), and no product is left to fuse into it.
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 sum2(float2 p, float2 q, float2 one) { return __ffma2_rn(q, one, p); }

__device__ __forceinline__ float lo_bf16(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float hi_bf16(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Two E4M3 codes (round to nearest even, saturated), a in the low byte.
__device__ __forceinline__ uint32_t e4m3x2(float a, float b)
{
    return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3)) & 0xFFFFu;
}

// c, s and -s of the lane's pairs pbase .. pbase + 7 (zero past n_rot) from
// the position's table row, packed two pairs at a time.
__device__ __forceinline__ void load_coeffs(const float *cs, int pbase, int half, int n_rot, float2 (&C)[4],
                                            float2 (&S)[4], float2 (&NS)[4])
{
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int i0 = 2 * i, i1 = 2 * i + 1;
        const float c0 = i0 < n_rot ? __ldg(cs + pbase + i0) : 0.0f;
        const float c1 = i1 < n_rot ? __ldg(cs + pbase + i1) : 0.0f;
        const float s0 = i0 < n_rot ? __ldg(cs + half + pbase + i0) : 0.0f;
        const float s1 = i1 < n_rot ? __ldg(cs + half + pbase + i1) : 0.0f;
        C[i] = make_float2(c0, c1);
        S[i] = make_float2(s0, s1);
        NS[i] = make_float2(-s0, -s1);
    }
}

// The lane's two 8-element chunks (element offsets in the head), its first
// pair index, and how many of its eight pairs rotate (8: all, 0: none).
template <int kL, bool kInterleaved>
__device__ __forceinline__ void lane_layout(int li, int rot_dim, int &off0, int &off1, int &pbase, int &n_rot)
{
    const int half = rot_dim >> 1;
    pbase = 8 * li;
    if (kInterleaved) {
        off0 = 16 * li;
        off1 = off0 + 8;
        n_rot = min(8, max(0, half - pbase));
    } else {
        const int npl = half >> 3;                 // rotating lanes
        if (li < npl) {
            off0 = 8 * li;
            off1 = half + 8 * li;
            n_rot = 8;
        } else {
            off0 = rot_dim + 16 * (li - npl);
            off1 = off0 + 8;
            n_rot = 0;
        }
    }
}

// One head's 16 elements in this lane (chunks w0, w1): rotation, the head's
// scale (a reduction over its kL lanes; every lane of the warp must call this
// together) and the codes, which are stored when `store`.
template <int kL, bool kInterleaved>
__device__ __forceinline__ void rope_head(const uint4 w0, const uint4 w1, const float2 (&C)[4], const float2 (&S)[4],
                                          const float2 (&NS)[4], float2 ONE, int n_rot, bool store, uint8_t *dst,
                                          int off0, int off1, float *scale_dst, int li)
{
    const uint32_t ww[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
    // (a'_0, a'_1) and (b'_0, b'_1) of the lane's pairs 2i, 2i + 1
    float2 A[4], B[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if (kInterleaved) {
            A[i] = make_float2(lo_bf16(ww[2 * i]), lo_bf16(ww[2 * i + 1]));
            B[i] = make_float2(hi_bf16(ww[2 * i]), hi_bf16(ww[2 * i + 1]));
        } else {
            A[i] = make_float2(lo_bf16(ww[i]), hi_bf16(ww[i]));
            B[i] = make_float2(lo_bf16(ww[4 + i]), hi_bf16(ww[4 + i]));
        }
    }
    // a = a' c + b' s, b = b' c + a' (-s), each product and the sum rounded
    float2 RA[4], RB[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        RA[i] = sum2(mul2(A[i], C[i]), mul2(B[i], S[i]), ONE);
        RB[i] = sum2(mul2(B[i], C[i]), mul2(A[i], NS[i]), ONE);
    }
    if (n_rot < 8) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if (2 * i >= n_rot) { RA[i].x = A[i].x; RB[i].x = B[i].x; }
            if (2 * i + 1 >= n_rot) { RA[i].y = A[i].y; RB[i].y = B[i].y; }
        }
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        amax = fmaxf(amax, fabsf(RA[i].x));
        amax = fmaxf(amax, fabsf(RA[i].y));
        amax = fmaxf(amax, fabsf(RB[i].x));
        amax = fmaxf(amax, fabsf(RB[i].y));
    }
#pragma unroll
    for (int o = kL / 2; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const bool fast = amax >= 0x1p-60f && amax <= 0x1p100f;
    const float sc = fast ? div448(amax) : (amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f);
    float2 QA[4], QB[4];
    if (fast) {
        // reciprocal refinement (see with_sign_of), two elements per instruction
        const float rs = __frcp_rn(sc);
        const float2 RS = make_float2(rs, rs), NSC = make_float2(-sc, -sc);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 qa = mul2(RA[i], RS), qb = mul2(RB[i], RS);
            const float2 ta = fma2(fma2(qa, NSC, RA[i]), RS, qa), tb = fma2(fma2(qb, NSC, RB[i]), RS, qb);
            QA[i] = make_float2(with_sign_of(ta.x, RA[i].x), with_sign_of(ta.y, RA[i].y));
            QB[i] = make_float2(with_sign_of(tb.x, RB[i].x), with_sign_of(tb.y, RB[i].y));
        }
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            QA[i] = make_float2(__fdiv_rn(RA[i].x, sc), __fdiv_rn(RA[i].y, sc));
            QB[i] = make_float2(__fdiv_rn(RB[i].x, sc), __fdiv_rn(RB[i].y, sc));
        }
    }
    // codes in element order: chunk 0 then chunk 1
    uint32_t c0[2], c1[2];
    if (kInterleaved) {
        // elements 4i .. 4i + 3 are a_2i, b_2i, a_2i+1, b_2i+1
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t wd = e4m3x2(QA[i].x, QB[i].x) | (e4m3x2(QA[i].y, QB[i].y) << 16);
            if (i < 2) c0[i] = wd;
            else c1[i - 2] = wd;
        }
    } else {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            c0[i] = e4m3x2(QA[2 * i].x, QA[2 * i].y) | (e4m3x2(QA[2 * i + 1].x, QA[2 * i + 1].y) << 16);
            c1[i] = e4m3x2(QB[2 * i].x, QB[2 * i].y) | (e4m3x2(QB[2 * i + 1].x, QB[2 * i + 1].y) << 16);
        }
    }
    if (store) {
        *reinterpret_cast<uint2 *>(dst + off0) = make_uint2(c0[0], c0[1]);
        *reinterpret_cast<uint2 *>(dst + off1) = make_uint2(c1[0], c1[1]);
        if (li == 0) *scale_dst = sc;
    }
}

// kP passes of 32 / kL heads from h00 on: this lane's two 16-byte chunks of
// each head (zeros past h_end), all loads issued before any is used.
template <int kL, int kP>
__device__ __forceinline__ void load_pass(uint4 (&w)[kP][2], const __nv_bfloat16 *__restrict__ x, long long row,
                                          int h00, int h_end, int sub, int off0, int off1)
{
    constexpr int kHd = 16 * kL, kHpw = 32 / kL;
#pragma unroll
    for (int u = 0; u < kP; ++u) {
        const int h = h00 + u * kHpw + sub;
        if (h < h_end) {
            const __nv_bfloat16 *src = x + (row + h) * kHd;
            w[u][0] = __ldg(reinterpret_cast<const uint4 *>(src + off0));
            w[u][1] = __ldg(reinterpret_cast<const uint4 *>(src + off1));
        } else {
            w[u][0] = w[u][1] = make_uint4(0u, 0u, 0u, 0u);
        }
    }
}

// Each head is handled by kL = head_dim / 16 lanes with 16 elements per lane,
// read as two 8-element chunks (two 16-byte loads), so that every rotary pair
// has both its elements in one lane:
//   neox pairs (i, i + rot_dim/2): a rotating lane holds the chunk of first
//     elements at 8 li and the chunk of their partners at rot_dim/2 + 8 li
//     (rot_dim a multiple of 16); the remaining lanes hold the passed-through
//     tail, 16 consecutive elements from rot_dim on;
//   interleaved pairs (2i, 2i + 1): lane li holds elements 16 li .. 16 li + 15,
//     eight pairs, each pair one bf16x2 word.
// A lane's eight pairs form four packs of two, (a'_0, a'_1) and (b'_0, b'_1),
// and the rotation a = a' c + b' s, b = b' c + a' (-s) takes three packed
// instructions per pack and output half; the quotient by the head's scale
// another three per pack.  A warp processes 32 / kL heads at once and takes
// one token and a chunk of hc of its heads per item: the token's position and
// the lane's rotary coefficients are loaded once for the chunk.  The loads of
// an item overlap: the next item's position is read while this one runs, and
// the first pass of head rows (which do not depend on the position) is
// requested before the coefficients.
template <int kL, bool kInterleaved>
__global__ void __launch_bounds__(256, 2) inv_rope_quant_kernel(const __nv_bfloat16 *__restrict__ x,
                                                             const int32_t *__restrict__ positions,
                                                             const float *__restrict__ cos_sin, int T, int n_heads,
                                                             int rot_dim, int max_pos, int hc, float one, uint8_t *q,
                                                             float *scales, int32_t *status)
{
    const float2 ONE = make_float2(one, one);      // 1.0, passed in (see sum2)
    constexpr int kHd = 16 * kL;
    constexpr int kHpw = 32 / kL;                  // heads per warp pass
    const int lane = threadIdx.x & 31;
    const int warp_g = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int n_warps = (gridDim.x * blockDim.x) >> 5;
    const int sub = lane / kL, li = lane % kL;     // head within the pass, lane within the head
    const int half = rot_dim >> 1;
    const int n_chunks = (n_heads + hc - 1) / hc;
    const long long n_items = static_cast<long long>(T) * n_chunks;
    int off0, off1, pbase, n_rot;
    lane_layout<kL, kInterleaved>(li, rot_dim, off0, off1, pbase, n_rot);
    constexpr int kP = 4;                          // passes whose loads are in flight together
    int p_next = warp_g < n_items ? __ldg(positions + static_cast<int>(warp_g / n_chunks)) : 0;
    for (long long item = warp_g; item < n_items; item += n_warps) {
        const int t = static_cast<int>(item / n_chunks);
        const int h_begin = static_cast<int>(item % n_chunks) * hc;
        const int h_end = min(n_heads, h_begin + hc);
        const int p = p_next;
        if (item + n_warps < n_items) p_next = __ldg(positions + static_cast<int>((item + n_warps) / n_chunks));
        const long long row = static_cast<long long>(t) * n_heads;
        uint4 w[kP][2];
        load_pass<kL, kP>(w, x, row, h_begin, h_end, sub, off0, off1);
        if (p < 0 || p >= max_pos) {                    // the same for the whole warp
            if (lane == 0 && status) set_status(status, MOE_ERR_DEVICE_CHECK);
            for (int h = h_begin + sub; h < h_end; h += kHpw) {
                if (li == 0) scales[row + h] = 0.0f;
                uint8_t *dst = q + (row + h) * kHd;
                *reinterpret_cast<uint2 *>(dst + off0) = make_uint2(0u, 0u);
                *reinterpret_cast<uint2 *>(dst + off1) = make_uint2(0u, 0u);
            }
            continue;
        }
        float2 C[4], S[4], NS[4];
        load_coeffs(cos_sin + static_cast<size_t>(p) * rot_dim, pbase, half, n_rot, C, S, NS);
        // kP passes of kHpw heads at a time (more bytes in flight per lane)
        for (int h00 = h_begin; h00 < h_end; h00 += kP * kHpw) {
            if (h00 != h_begin) load_pass<kL, kP>(w, x, row, h00, h_end, sub, off0, off1);
#pragma unroll
            for (int u = 0; u < kP; ++u) {
                const int h = h00 + u * kHpw + sub;
                if (h00 + u * kHpw >= h_end) break;        // uniform across the warp
                rope_head<kL, kInterleaved>(w[u][0], w[u][1], C, S, NS, ONE, n_rot, h < h_end, q + (row + h) * kHd, off0,
                                            off1, scales + row + h, li);
            }
        }
    }
}

}  // namespace moe

using namespace moe;

// Blocks of 256 threads of one kernel variant that fit on the whole GPU at
// once, cached per variant and device.
template <int kL, bool kInterleaved>
static int rope_resident_blocks()
{
    static std::atomic<int> cache[64];
    int dev = 0;
    cudaGetDevice(&dev);
    int n = (dev >= 0 && dev < 64) ? cache[dev].load(std::memory_order_relaxed) : 0;
    if (n == 0) {
        int sms = 0, per_sm = 0;
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, inv_rope_quant_kernel<kL, kInterleaved>, 256, 0);
        n = (sms > 0 ? sms : 148) * (per_sm > 0 ? per_sm : 1);
        if (dev >= 0 && dev < 64) cache[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

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
    const int L = s.head_dim / 16;
    const int hpw = 32 / L;
    // heads per warp item: all of a token's heads when there are enough tokens
    // to give every SM 32 warps, else fewer so that small batches still spread
    // over the GPU
    int hc = s.n_heads;
    while (hc > hpw && static_cast<long long>(s.num_tokens) * ((s.n_heads + hc - 1) / hc) < 148LL * 32)
        hc = ((hc / 2) + hpw - 1) / hpw * hpw;
    const long long items = static_cast<long long>(s.num_tokens) * ((s.n_heads + hc - 1) / hc);
    const long long want = (items + 7) / 8;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const __nv_bfloat16 *xb = static_cast<const __nv_bfloat16 *>(x);
    // one wave of resident blocks, each warp striding over the items
#define MOE_ROPE(LL, IL)                                                                                     \
    do {                                                                                                     \
        const long long cap = static_cast<long long>(rope_resident_blocks<LL, IL>());                      \
        const int blocks = static_cast<int>(want < cap ? want : cap);                                        \
        inv_rope_quant_kernel<LL, IL><<<blocks, 256, 0, st>>>(xb, positions, cos_sin, s.num_tokens,          \
                                                               s.n_heads, s.rot_dim, s.max_pos, hc, 1.0f, q,  \
                                                               scales, status);                              \
    } while (0)
    if (s.interleaved) {
        if (L == 4) MOE_ROPE(4, true);
        else if (L == 8) MOE_ROPE(8, true);
        else MOE_ROPE(16, true);
    } else {
        if (L == 4) MOE_ROPE(4, false);
        else if (L == 8) MOE_ROPE(8, false);
        else MOE_ROPE(16, false);
    }
#undef MOE_ROPE
    launches = 1;
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
