// small_kernels.cu - the memory-bound steps of the fused-MoE layer:
//   routing (top-k gating), alignment/permutation, gather (+E4M3 quantisation)
//   and the weighted combine.
// The AWS post ("Mixture-of-Experts kernel engineering on Amazon SageMaker AI",
// abstract) names these steps as token routing, data shuffling and expert
// aggregation; the Chinese retelling (section "2. 用于FP8量化的Triton后端路由")
// stresses keeping routing decisions on the GPU, without host-side control
// flow.  Nothing here reads a routing result on the host.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "common.cuh"

namespace moe {

// ------------------------------------------------------------------ routing
// Order-preserving map of a float logit to an unsigned key: larger logit ->
// larger key, -0 == +0, NaN below -inf (key 0).
__device__ __forceinline__ uint32_t logit_key(float v)
{
    if (v != v) return 0u;
    if (v == 0.0f) v = 0.0f;
    uint32_t u = __float_as_uint(v);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Top-k of one token by one warp.  Lane l holds logits l, l+32, ...; the k
// winners are found by k rounds of a warp-wide arg-max over the 64-bit key
// (logit key, ~expert id): larger logit first, ties to the lower id.
template <int kSlots>
__device__ __forceinline__ void route_warp(const float *l, int E, int k, int gate, int renorm,
                                           float routed_scale, int32_t *ids_t, float *w_t, int lane)
{
    uint64_t key[kSlots];
    uint32_t taken = 0;
#pragma unroll
    for (int i = 0; i < kSlots; ++i) {
        const int e = i * 32 + lane;
        if (e < E) {
            key[i] = (static_cast<uint64_t>(logit_key(l[e])) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(e));
        } else {
            key[i] = 0;
            taken |= 1u << i;
        }
    }
    int my_id = -1;
    for (int j = 0; j < k; ++j) {
        uint64_t best = 0;
#pragma unroll
        for (int i = 0; i < kSlots; ++i)
            if (!((taken >> i) & 1u) && key[i] > best) best = key[i];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const uint64_t other = __shfl_xor_sync(0xffffffffu, best, o);
            best = other > best ? other : best;
        }
        const int id = static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(best & 0xFFFFFFFFu));
        if ((id & 31) == lane) taken |= 1u << (id >> 5);
        if (lane == j) my_id = id;
    }
    const bool mine = lane < k;
    const float v = mine ? l[my_id] : 0.0f;
    float wt;
    if (gate == MOE_GATE_SOFTMAX) {
        if (renorm) {
            const float m = __shfl_sync(0xffffffffu, v, 0);
            const float ex = mine ? expf(v - m) : 0.0f;
            wt = ex / warp_sum(ex);
        } else {
            float m = -INFINITY;
            for (int e = lane; e < E; e += 32) m = fmaxf(m, l[e]);
            m = warp_max(m);
            float z = 0.0f;
            for (int e = lane; e < E; e += 32) z += expf(l[e] - m);
            z = warp_sum(z);
            wt = expf(v - m) / z;
        }
    } else {
        const float s = mine ? 1.0f / (1.0f + expf(-v)) : 0.0f;
        wt = renorm ? s / warp_sum(s) : s;
    }
    if (mine) {
        ids_t[lane] = my_id;
        w_t[lane] = wt * routed_scale;
    }
}

// One warp per token.  As the first kernel of the fused layer it also clears
// `n_zero` words at `zero` (the control words and counters the later kernels
// use after their dependency waits); nothing in this kernel reads them.
template <int kSlots>
__global__ void __launch_bounds__(256) route_topk_kernel(const float *__restrict__ logits, int T,
                                                         int E, int k, int gate, int renorm,
                                                         float routed_scale, int32_t *ids,
                                                         float *w, int32_t *zero, int n_zero)
{
    grid_dep_wait();
    grid_dep_launch();
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n_zero; i += gridDim.x * blockDim.x) zero[i] = 0;
    const int lane = threadIdx.x & 31;
    const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (t >= T) return;
    route_warp<kSlots>(logits + static_cast<size_t>(t) * E, E, k, gate, renorm, routed_scale,
                       ids + static_cast<size_t>(t) * k, w + static_cast<size_t>(t) * k, lane);
}

cudaError_t launch_route(const moe_shape_t &s, const float *logits, int32_t *ids, float *w,
                         cudaStream_t st, int32_t *zero, int n_zero, bool chained)
{
    const int threads = 256, blocks = (s.T * 32 + threads - 1) / threads;
    const int slots = (s.E + 31) / 32;
#define MOE_ROUTE(N)                                                                                            \
    return launch_kernel(route_topk_kernel<N>, dim3(blocks), dim3(threads), 0, st, chained, logits, s.T, s.E, s.k, \
                         s.gate, s.renorm, s.routed_scale, ids, w, zero, n_zero)
    if (slots <= 1) MOE_ROUTE(1);
    if (slots <= 2) MOE_ROUTE(2);
    if (slots <= 4) MOE_ROUTE(4);
    if (slots <= 8) MOE_ROUTE(8);
    MOE_ROUTE(16);
#undef MOE_ROUTE
}

// ------------------------------------------------------------------ router
// Router logits and top-k in one launch (the step before routing; the Chinese
// retelling, section "2. 用于FP8量化的Triton后端路由", keeps routing inside
// the fused kernel).  l[t,e] = sum_h x[t,h] * Wg[e,h] in a fixed order, so
// that the result does not depend on the launch shape:
//   lane l of a warp sums in double, in ascending h, the products of the
//   8-element chunks c (16-byte loads) with c mod 32 == l; the warp combines
//   its 32 partial sums by s_l += s_(l xor o), o = 16, 8, 4, 2, 1; the sum is
//   rounded once to fp32.
// Block (t, g) computes token t's logits of experts [32 g, 32 g + 32): warp
// w takes experts 32 g + 4 w .. 32 g + 4 w + 3 together (four independent
// accumulation chains per lane, one load of x for four rows of Wg; the order
// within each chain is the one above).  The last block of token t to finish
// (ticket) selects its top-k from all E logits, as route_topk_kernel does.
__device__ __forceinline__ double dot8(uint4 a, uint4 b, double acc)
{
    const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        acc = fma(static_cast<double>(__uint_as_float(wa[i] << 16)),
                  static_cast<double>(__uint_as_float(wb[i] << 16)), acc);      // exact product
        acc = fma(static_cast<double>(__uint_as_float(wa[i] & 0xFFFF0000u)),
                  static_cast<double>(__uint_as_float(wb[i] & 0xFFFF0000u)), acc);
    }
    return acc;
}

template <int kSlots>
__global__ void __launch_bounds__(256) router_topk_kernel(const uint4 *__restrict__ x, const uint4 *__restrict__ wg,
                                                          int H, int E, int k, int gate, int renorm,
                                                          float routed_scale, float *logits, int32_t *tickets,
                                                          int32_t *ids, float *w)
{
    grid_dep_wait();
    grid_dep_launch();
    __shared__ float s_l[kMaxExperts];
    __shared__ int s_last;
    const int t = blockIdx.x, g = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nc = H / 8;
    const uint4 *xr = x + static_cast<size_t>(t) * nc;
    constexpr int kPer = 4;                      // experts per warp
    const int e0 = g * 32 + warp * kPer;
    if (e0 < E) {
        const uint4 *wr[kPer];
#pragma unroll
        for (int q = 0; q < kPer; ++q)             // rows past E repeat the last one (not stored)
            wr[q] = wg + static_cast<size_t>(min(e0 + q, E - 1)) * nc;
        double acc[kPer];
#pragma unroll
        for (int q = 0; q < kPer; ++q) acc[q] = 0.0;
        for (int c = lane; c < nc; c += 32) {
            const uint4 a = __ldg(xr + c);
#pragma unroll
            for (int q = 0; q < kPer; ++q) acc[q] = dot8(a, __ldg(wr[q] + c), acc[q]);
        }
#pragma unroll
        for (int q = 0; q < kPer; ++q) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc[q] += __shfl_xor_sync(0xffffffffu, acc[q], o);
            if (lane == 0 && e0 + q < E) logits[static_cast<size_t>(t) * E + e0 + q] = __double2float_rn(acc[q]);
        }
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(&tickets[t], 1) == static_cast<int>(gridDim.y) - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    for (int e = threadIdx.x; e < E; e += blockDim.x) s_l[e] = __ldcg(&logits[static_cast<size_t>(t) * E + e]);
    __syncthreads();
    if (warp == 0)
        route_warp<kSlots>(s_l, E, k, gate, renorm, routed_scale, ids + static_cast<size_t>(t) * k,
                           w + static_cast<size_t>(t) * k, lane);
}

cudaError_t launch_router(const moe_shape_t &s, const void *x, const void *wg, float *logits,
                          int32_t *tickets, int32_t *ids, float *w, cudaStream_t st, bool chained)
{
    const dim3 grid(s.T, (s.E + 31) / 32);
    const int slots = (s.E + 31) / 32;
    const uint4 *xv = static_cast<const uint4 *>(x), *wv = static_cast<const uint4 *>(wg);
#define MOE_ROUTER(N)                                                                                  \
    return launch_kernel(router_topk_kernel<N>, grid, dim3(256), 0, st, chained, xv, wv, s.H, s.E, s.k, \
                         s.gate, s.renorm, s.routed_scale, logits, tickets, ids, w)
    if (slots <= 1) MOE_ROUTER(1);
    if (slots <= 2) MOE_ROUTER(2);
    if (slots <= 4) MOE_ROUTER(4);
    if (slots <= 8) MOE_ROUTER(8);
    MOE_ROUTER(16);
#undef MOE_ROUTER
}

// ------------------------------------------------------------------ align
// Block b counts the expert ids of routed rows [b*1024, (b+1)*1024) into a
// shared histogram (integer atomics: the counts do not depend on order).  The
// last block to finish (ticket) turns the per-block histograms into counts,
// padded segment offsets and each block's first slot per expert, fills pad
// slots with -1 and writes the shared experts' rows.
__global__ void __launch_bounds__(1024) align_count_kernel(
    const int32_t *__restrict__ ids, int R, int T, int E, int n_shared, int pad,
    int32_t *chunk_hist, int32_t *chunk_base, int32_t *counts, int32_t *offsets,
    int32_t *sorted_rows, Ctrl *ctrl)
{
    grid_dep_wait();
    grid_dep_launch();
    extern __shared__ int32_t sh[];
    __shared__ int s_last;
    const int Et = E + n_shared;
    const int tid = threadIdx.x, nb = gridDim.x;
    for (int i = tid; i < Et; i += blockDim.x) sh[i] = 0;
    __syncthreads();
    const int f = blockIdx.x * kAlignChunk + tid;
    if (f < R) {
        const int e = ids[f];
        if (e >= 0 && e < E) atomicAdd(&sh[e], 1);
        else set_status(&ctrl->status, MOE_ERR_DEVICE_CHECK);
    }
    __syncthreads();
    for (int i = tid; i < Et; i += blockDim.x) chunk_hist[static_cast<size_t>(blockIdx.x) * Et + i] = sh[i];
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = (atomicAdd(&ctrl->ticket, 1) == nb - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    // totals and padded sizes
    for (int e = tid; e < Et; e += blockDim.x) {
        int c = 0;
        if (e < E)
            for (int b = 0; b < nb; ++b) c += __ldcg(&chunk_hist[static_cast<size_t>(b) * Et + e]);
        else
            c = T;
        counts[e] = c;
        sh[e] = (c + pad - 1) / pad * pad;
    }
    __syncthreads();
    // exclusive scan of the padded sizes by warp 0 (contiguous chunk per lane)
    if (tid < 32) {
        const int per = (Et + 31) / 32;
        const int lo = min(Et, tid * per), hi = min(Et, lo + per);
        int sum = 0;
        for (int e = lo; e < hi; ++e) sum += sh[e];
        int inc = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, inc, o);
            if (tid >= o) inc += v;
        }
        int run = inc - sum;
        for (int e = lo; e < hi; ++e) {
            const int sz = sh[e];
            offsets[e] = run;
            sh[e] = run;
            run += sz;
        }
        if (tid == 31) offsets[Et] = inc;
    }
    __syncthreads();
    // first slot of each (block, expert) pair, pad slots, shared experts
    for (int e = tid; e < Et; e += blockDim.x) {
        const int start = sh[e];
        if (e < E) {
            int base = start;
            for (int b = 0; b < nb; ++b) {
                chunk_base[static_cast<size_t>(b) * Et + e] = base;
                base += __ldcg(&chunk_hist[static_cast<size_t>(b) * Et + e]);
            }
        }
        const int c = counts[e];
        const int end = start + (c + pad - 1) / pad * pad;
        for (int q = start + c; q < end; ++q) sorted_rows[q] = -1;
    }
    for (int s = 0; s < n_shared; ++s)
        for (int t = tid; t < T; t += blockDim.x) sorted_rows[sh[E + s] + t] = R + s * T + t;
    if (tid == 0) ctrl->ticket = 0;
}

// Each block places its 1024 routed rows: rank within the warp by
// __match_any_sync, ranks of earlier warps by a prefix over per-warp counts,
// plus the block's first slot for that expert.  The result is the stable
// (ascending row index) order within every expert, independent of timing.
__global__ void __launch_bounds__(1024) align_scatter_kernel(const int32_t *__restrict__ ids,
                                                             int R, int E, int Et,
                                                             const int32_t *chunk_base,
                                                             int32_t *sorted_rows, int32_t *inv)
{
    grid_dep_wait();
    grid_dep_launch();
    extern __shared__ int32_t wc[];   // [32 warps][Et]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int i = tid; i < 32 * Et; i += blockDim.x) wc[i] = 0;
    __syncthreads();
    const int f = blockIdx.x * kAlignChunk + tid;
    int e = f < R ? ids[f] : -1;
    const bool valid = e >= 0 && e < E;
    if (!valid) e = -1;
    const unsigned same = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(same & ((1u << lane) - 1u));
    if (valid && rank == 0) wc[warp * Et + e] = __popc(same);
    __syncthreads();
    for (int x = tid; x < Et; x += blockDim.x) {
        int run = 0;
        for (int q = 0; q < 32; ++q) {
            const int c = wc[q * Et + x];
            wc[q * Et + x] = run;
            run += c;
        }
    }
    __syncthreads();
    if (f < R) {
        if (valid) {
            const int slot = chunk_base[static_cast<size_t>(blockIdx.x) * Et + e] + wc[warp * Et + e] + rank;
            sorted_rows[slot] = f;
            inv[f] = slot;
        } else {
            inv[f] = -1;
        }
    }
}

// All routed rows in one block (R <= 1024, every decode batch here): count,
// scan, pad and place, with the histogram, the offsets and the per-warp counts
// in shared memory sm_al [33 * Et].  Same result as the two-kernel path.
// `ids` may live in global or shared memory; the whole block calls this.
__device__ __forceinline__ void align_block(const int32_t *ids, int R, int T, int E, int n_shared, int pad,
                                            int32_t *counts, int32_t *offsets, int32_t *sorted_rows,
                                            int32_t *inv, Ctrl *ctrl, int32_t *sm_al)
{
    const int Et = E + n_shared;
    int32_t *hist = sm_al;                 // [Et]: counts, then segment starts
    int32_t *wc = sm_al + Et;              // [32 warps][Et]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int i = tid; i < Et * 33; i += blockDim.x) sm_al[i] = 0;
    __syncthreads();
    const int f = tid;
    int e = f < R ? ids[f] : -1;
    const bool valid = e >= 0 && e < E;
    if (f < R && !valid) set_status(&ctrl->status, MOE_ERR_DEVICE_CHECK);
    if (!valid) e = -1;
    const unsigned same = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(same & ((1u << lane) - 1u));
    if (valid && rank == 0) {
        wc[warp * Et + e] = __popc(same);
        atomicAdd(&hist[e], __popc(same));
    }
    __syncthreads();
    for (int x = tid; x < Et; x += blockDim.x) {
        const int c = x < E ? hist[x] : T;
        counts[x] = c;
        hist[x] = (c + pad - 1) / pad * pad;
        int run = 0;                                     // exclusive prefix over warps
        for (int q = 0; q < 32; ++q) {
            const int v = wc[q * Et + x];
            wc[q * Et + x] = run;
            run += v;
        }
    }
    __syncthreads();
    if (tid < 32) {                                      // exclusive scan of padded sizes
        const int per = (Et + 31) / 32;
        const int lo = min(Et, tid * per), hi = min(Et, lo + per);
        int sum = 0;
        for (int x = lo; x < hi; ++x) sum += hist[x];
        int inc = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, inc, o);
            if (tid >= o) inc += v;
        }
        int run = inc - sum;
        for (int x = lo; x < hi; ++x) {
            const int sz = hist[x];
            offsets[x] = run;
            hist[x] = run;
            run += sz;
        }
        if (tid == 31) offsets[Et] = inc;
    }
    __syncthreads();
    for (int x = tid; x < Et; x += blockDim.x) {         // pad slots
        const int start = hist[x], c = counts[x];
        const int end = start + (c + pad - 1) / pad * pad;
        for (int q = start + c; q < end; ++q) sorted_rows[q] = -1;
    }
    for (int sh = 0; sh < n_shared; ++sh)
        for (int t = tid; t < T; t += blockDim.x) sorted_rows[hist[E + sh] + t] = R + sh * T + t;
    if (f < R) {
        if (valid) {
            const int slot = hist[e] + wc[warp * Et + e] + rank;
            sorted_rows[slot] = f;
            inv[f] = slot;
        } else {
            inv[f] = -1;
        }
    }
}

__global__ void __launch_bounds__(1024) align_single_kernel(const int32_t *__restrict__ ids, int R, int T,
                                                            int E, int n_shared, int pad, int32_t *counts,
                                                            int32_t *offsets, int32_t *sorted_rows,
                                                            int32_t *inv, Ctrl *ctrl)
{
    grid_dep_wait();
    grid_dep_launch();
    extern __shared__ int32_t sm_al[];
    align_block(ids, R, T, E, n_shared, pad, counts, offsets, sorted_rows, inv, ctrl, sm_al);
}

// Routing and alignment of a decode batch in one block (R = T*k <= 1024), the
// first kernel of the fused layer: it also clears the status word, the align
// ticket, the GEMMs' stream-K tile counters and the fused combine's arrival
// counters (`zero`, `n_zero` words), which the later kernels of the call use
// only after their dependency waits.  Warp w
// routes tokens w, w + 32, ... (as route_topk_kernel); the ids stay in shared
// memory for the alignment.
template <int kSlots>
__global__ void __launch_bounds__(1024) route_align_kernel(const float *__restrict__ logits, int T, int E, int k,
                                                           int gate, int renorm, float routed_scale, int n_shared,
                                                           int pad, float *w, int32_t *counts, int32_t *offsets,
                                                           int32_t *sorted_rows, int32_t *inv, Ctrl *ctrl,
                                                           int32_t *zero, int n_zero)
{
    grid_dep_wait();
    grid_dep_launch();
    __shared__ int32_t s_ids[kAlignChunk];
    extern __shared__ int32_t sm_al[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < n_zero; i += blockDim.x) zero[i] = 0;
    __syncthreads();                                     // status cleared before anything can set it
    for (int t = warp; t < T; t += blockDim.x >> 5)
        route_warp<kSlots>(logits + static_cast<size_t>(t) * E, E, k, gate, renorm, routed_scale, s_ids + t * k,
                           w + static_cast<size_t>(t) * k, lane);
    __syncthreads();
    align_block(s_ids, T * k, T, E, n_shared, pad, counts, offsets, sorted_rows, inv, ctrl, sm_al);
}

cudaError_t launch_route_align(const moe_shape_t &s, const float *logits, float *w, int32_t *counts,
                               int32_t *offsets, int32_t *sorted_rows, int32_t *inv, Ctrl *ctrl, int32_t *zero,
                               int n_zero, cudaStream_t st, bool chained)
{
    const int Et = s.E + s.n_shared;
    const int slots = (s.E + 31) / 32;
    static PerDeviceOnce attrs;
    attrs([] {
        cudaFuncSetAttribute(route_align_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, 33 * kMaxExpertsTotal * 4);
        cudaFuncSetAttribute(route_align_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, 33 * kMaxExpertsTotal * 4);
        cudaFuncSetAttribute(route_align_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, 33 * kMaxExpertsTotal * 4);
        cudaFuncSetAttribute(route_align_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, 33 * kMaxExpertsTotal * 4);
        cudaFuncSetAttribute(route_align_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, 33 * kMaxExpertsTotal * 4);
    });
    const size_t smem = 33 * Et * sizeof(int32_t);
#define MOE_RA(N)                                                                                                  \
    return launch_kernel(route_align_kernel<N>, dim3(1), dim3(kAlignChunk), smem, st, chained, logits, s.T, s.E, \
                         s.k, s.gate, s.renorm, s.routed_scale, s.n_shared, s.pad, w, counts, offsets, sorted_rows, \
                         inv, ctrl, zero, n_zero)
    if (slots <= 1) MOE_RA(1);
    if (slots <= 2) MOE_RA(2);
    if (slots <= 4) MOE_RA(4);
    if (slots <= 8) MOE_RA(8);
    MOE_RA(16);
#undef MOE_RA
}

cudaError_t launch_align(const moe_shape_t &s, const int32_t *ids, int32_t *counts,
                         int32_t *offsets, int32_t *sorted_rows, int32_t *inv, int32_t *chunk_hist,
                         int32_t *chunk_base, Ctrl *ctrl, cudaStream_t st, int *launches, bool chained,
                         bool ticket_zero)
{
    const int R = s.T * s.k, Et = s.E + s.n_shared;
    const int nb = (R + kAlignChunk - 1) / kAlignChunk;
    static PerDeviceOnce attrs;
    attrs([] {
        cudaFuncSetAttribute(align_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             32 * kMaxExpertsTotal * 4);
        cudaFuncSetAttribute(align_single_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             33 * kMaxExpertsTotal * 4);
    });
    if (nb == 1) {
        *launches += 1;
        return launch_kernel(align_single_kernel, dim3(1), dim3(kAlignChunk), 33 * Et * sizeof(int32_t), st,
                             chained, ids, R, s.T, s.E, s.n_shared, s.pad, counts, offsets, sorted_rows, inv,
                             ctrl);
    }
    if (!chained && !ticket_zero) {
        cudaError_t err = cudaMemsetAsync(&ctrl->ticket, 0, sizeof(int32_t), st);
        if (err != cudaSuccess) return err;
    }
    cudaError_t err = launch_kernel(align_count_kernel, dim3(nb), dim3(kAlignChunk), Et * sizeof(int32_t), st,
                                    chained, ids, R, s.T, s.E, s.n_shared, s.pad, chunk_hist, chunk_base,
                                    counts, offsets, sorted_rows, ctrl);
    if (err != cudaSuccess) return err;
    *launches += 2;
    return launch_kernel(align_scatter_kernel, dim3(nb), dim3(kAlignChunk), 32 * Et * sizeof(int32_t), st,
                         chained, ids, R, s.E, Et, static_cast<const int32_t *>(chunk_base), sorted_rows, inv);
}

// ------------------------------------------------------------------ gather
// One warp per slot of the permuted buffer, 16-byte vectors along the row.
// skip_pad: leave pad slots unwritten (inside the fused layer, where a pad
// slot's row reaches no real output: an MMA column depends only on its own
// operand row, and the combine skips pad slots); else write zeros there.
template <bool kQuant>
__global__ void __launch_bounds__(256) gather_kernel(const uint4 *__restrict__ x,
                                                     const int32_t *__restrict__ sorted_rows,
                                                     const int32_t *__restrict__ offsets, int Et,
                                                     int T, int k, int H, float a1, void *xp, int skip_pad)
{
    grid_dep_wait();
    grid_dep_launch();
    const int lane = threadIdx.x & 31;
    const int nvec = H / 8;                       // 8 bf16 per 16 bytes
    const int nchunk = (nvec + 31) / 32;          // 512-byte chunks per row
    const int total = offsets[Et];
    const int R = T * k;
    for (long long item = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; item < static_cast<long long>(total) * nchunk;
         item += (gridDim.x * blockDim.x) >> 5) {
        const int s = static_cast<int>(item / nchunk);
        const int v = static_cast<int>(item % nchunk) * 32 + lane;
        const int f = sorted_rows[s];
        const int t = f < 0 ? -1 : (f < R ? f / k : (f - R) % T);
        if (v >= nvec || (t < 0 && skip_pad)) continue;
        if (!kQuant) {
            uint4 *dst = reinterpret_cast<uint4 *>(xp) + static_cast<size_t>(s) * nvec;
            const uint4 *src = x + static_cast<size_t>(t < 0 ? 0 : t) * nvec;
            dst[v] = t < 0 ? make_uint4(0, 0, 0, 0) : __ldg(src + v);
        } else {
            uint2 *dst = reinterpret_cast<uint2 *>(xp) + static_cast<size_t>(s) * nvec;
            const uint4 *src = x + static_cast<size_t>(t < 0 ? 0 : t) * nvec;
            if (t < 0) {
                dst[v] = make_uint2(0, 0);
            } else {
                const uint4 d = __ldg(src + v);
                const uint32_t wv[4] = {d.x, d.y, d.z, d.w};
                uint32_t q[2] = {0, 0};
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint32_t bits = (wv[i >> 1] >> ((i & 1) * 16)) & 0xFFFFu;
                    const float val = __uint_as_float(bits << 16) / a1;
                    const uint32_t c = __nv_cvt_float_to_fp8(val, __NV_SATFINITE, __NV_E4M3);
                    q[i >> 2] |= (c & 0xFFu) << ((i & 3) * 8);
                }
                dst[v] = make_uint2(q[0], q[1]);
            }
        }
    }
}

cudaError_t launch_gather(const moe_shape_t &s, const void *x, const int32_t *sorted_rows,
                          const int32_t *offsets, float a1, void *xp, int64_t max_rows,
                          cudaStream_t st, bool chained, bool skip_pad)
{
    const int Et = s.E + s.n_shared;
    const int64_t warps = max_rows * ((s.H / 8 + 31) / 32);
    int blocks = static_cast<int>((warps + 7) / 8);
    if (blocks > 148 * 16) blocks = 148 * 16;
    if (blocks < 1) blocks = 1;
    return launch_kernel(s.adtype == MOE_E4M3 ? gather_kernel<true> : gather_kernel<false>, dim3(blocks),
                         dim3(256), 0, st, chained, static_cast<const uint4 *>(x), sorted_rows, offsets, Et,
                         s.T, s.k, s.H, a1, xp, skip_pad ? 1 : 0);
}

// ------------------------------------------------------------------ hi/lo split
// E4M3 weights with bf16 activations run on the E4M3 tensor path.  Each
// activation row v (bf16, K values) is written as two E4M3 planes under one
// power-of-two scale s per row:
//   hi = e4m3(v / s),  lo = e4m3(v / s - hi),  v = s * (hi + lo).
// s is the smallest power of two with max|v| <= 448 s, so nothing saturates.
// A bf16 value has 8 significant bits and hi keeps the top 4 (rounded), so
// the remainder v/s - hi needs at most 4 bits and is exact in E4M3 whenever
// it is at least 2^-6 (the smallest normal); smaller remainders round to the
// 2^-9 subnormal grid.  The split is therefore exact except for elements
// below about 2^-11 of the row's max magnitude, which are off by at most
// 2^-10 s (about 4.4e-6 of the row max): far below the bf16 rounding of
// the GEMM outputs.  Products of E4M3 codes are exact in the fp32
// accumulator, so the GEMM computes the bf16-activation products.
__device__ __forceinline__ float e4m3_value(uint32_t code)
{
    const __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(code), __NV_E4M3);
    return __half2float(__half(h));
}

__device__ __forceinline__ void split8(uint4 d, float inv_s, uint2 &hi, uint2 &lo)
{
    const uint32_t wv[4] = {d.x, d.y, d.z, d.w};
    uint32_t qh[2] = {0, 0}, ql[2] = {0, 0};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float v = __uint_as_float(((wv[i >> 1] >> ((i & 1) * 16)) & 0xFFFFu) << 16) * inv_s;
        const uint32_t ch = __nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3) & 0xFFu;
        const uint32_t cl = __nv_cvt_float_to_fp8(v - e4m3_value(ch), __NV_SATFINITE, __NV_E4M3) & 0xFFu;
        qh[i >> 2] |= ch << ((i & 3) * 8);
        ql[i >> 2] |= cl << ((i & 3) * 8);
    }
    hi = make_uint2(qh[0], qh[1]);
    lo = make_uint2(ql[0], ql[1]);
}

__device__ __forceinline__ float abs_max8(uint4 d)
{
    const uint32_t wv[4] = {d.x, d.y, d.z, d.w};
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        m = fmaxf(m, fabsf(__uint_as_float(wv[i] << 16)));
        m = fmaxf(m, fabsf(__uint_as_float(wv[i] & 0xFFFF0000u)));
    }
    return m;
}

// Exponent e of the row scale s = 2^e: amax = M * 2^E with M in [1, 2);
// amax <= 448 * 2^e  <=>  e >= E - 8 when M <= 1.75, else e >= E - 7.
__device__ __forceinline__ int row_scale_exp(float amax)
{
    const uint32_t b = __float_as_uint(amax);
    const int ef = static_cast<int>((b >> 23) & 0xFFu);
    if (ef == 0) return -126;                         // zero or subnormal max: any scale
    const int e = (ef - 127) - 8 + ((b & 0x7FFFFFu) > 0x600000u ? 1 : 0);
    return e < -126 ? -126 : e;
}

// Split one bf16 row of nv 16-byte vectors into its hi/lo planes and scale,
// the whole block cooperating.  A row of up to kRowRegs vectors per thread
// (K <= 8192 for 256 threads) is read once and kept in registers; a longer
// row is read twice (once for the max magnitude, once to split).
constexpr int kRowRegs = 4;
__device__ __forceinline__ void split_row(const uint4 *__restrict__ r, int nv, uint2 *ph, uint2 *pl, float *scale_out,
                                          float *s_red)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool in_regs = nv <= kRowRegs * static_cast<int>(blockDim.x);
    uint4 d[kRowRegs];
    float m = 0.0f;
    if (in_regs) {
#pragma unroll
        for (int i = 0; i < kRowRegs; ++i) {
            const int v = threadIdx.x + i * blockDim.x;
            if (v < nv) {
                d[i] = __ldg(r + v);
                m = fmaxf(m, abs_max8(d[i]));
            }
        }
    } else {
        for (int v = threadIdx.x; v < nv; v += blockDim.x) m = fmaxf(m, abs_max8(__ldg(r + v)));
    }
    m = warp_max(m);
    if (lane == 0) s_red[warp] = m;
    __syncthreads();
    m = s_red[0];
    for (int i = 1; i < static_cast<int>(blockDim.x >> 5); ++i) m = fmaxf(m, s_red[i]);
    __syncthreads();                                  // s_red is rewritten by the next row
    const int e = row_scale_exp(m);
    const float inv_s = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);   // 2^-e
    if (in_regs) {
#pragma unroll
        for (int i = 0; i < kRowRegs; ++i) {
            const int v = threadIdx.x + i * blockDim.x;
            if (v < nv) {
                uint2 hi, lo;
                split8(d[i], inv_s, hi, lo);
                ph[v] = hi;
                pl[v] = lo;
            }
        }
    } else {
        for (int v = threadIdx.x; v < nv; v += blockDim.x) {
            uint2 hi, lo;
            split8(__ldg(r + v), inv_s, hi, lo);
            ph[v] = hi;
            pl[v] = lo;
        }
    }
    if (threadIdx.x == 0) *scale_out = __uint_as_float(static_cast<uint32_t>(127 + e) << 23);
}

// One block per permuted row (grid-stride over the rows that exist).  With
// sorted_rows (inside the fused layer) pad slots are skipped: their rows
// reach no real output.
__global__ void __launch_bounds__(256) split_hilo_kernel(const uint4 *__restrict__ src, int K,
                                                         const int32_t *__restrict__ offsets, int Et,
                                                         int64_t lo_rows, uint2 *planes, float *scale,
                                                         const int32_t *__restrict__ sorted_rows)
{
    grid_dep_wait();
    grid_dep_launch();
    __shared__ float s_red[8];
    const int total = offsets[Et];
    const int nv = K / 8;
    for (int row = blockIdx.x; row < total; row += gridDim.x) {
        if (sorted_rows && sorted_rows[row] < 0) continue;       // the same for the whole block
        split_row(src + static_cast<size_t>(row) * nv, nv, planes + static_cast<size_t>(row) * nv,
                  planes + static_cast<size_t>(lo_rows + row) * nv, scale + row, s_red);
    }
}

// The gather and the hi/lo split in one pass (the fused layer with E4M3
// weights and bf16 activations): block per slot, the slot's token row read
// from x, its planes and scale written as split_hilo_kernel writes them.  Pad
// slots are skipped (their rows reach no real output).
__global__ void __launch_bounds__(256) gather_split_kernel(const uint4 *__restrict__ x,
                                                           const int32_t *__restrict__ sorted_rows,
                                                           const int32_t *__restrict__ offsets, int Et, int T,
                                                           int k, int H, int64_t lo_rows, uint2 *planes,
                                                           float *scale)
{
    grid_dep_wait();
    grid_dep_launch();
    __shared__ float s_red[8];
    const int total = offsets[Et];
    const int nv = H / 8;
    const int R = T * k;
    for (int row = blockIdx.x; row < total; row += gridDim.x) {
        const int f = sorted_rows[row];
        if (f < 0) continue;                                    // the same for the whole block
        const int t = f < R ? f / k : (f - R) % T;
        split_row(x + static_cast<size_t>(t) * nv, nv, planes + static_cast<size_t>(row) * nv,
                  planes + static_cast<size_t>(lo_rows + row) * nv, scale + row, s_red);
    }
}

cudaError_t launch_gather_split(const moe_shape_t &s, const void *x, const int32_t *sorted_rows,
                                const int32_t *offsets, void *planes, float *scale, int64_t max_rows,
                                cudaStream_t st, bool chained)
{
    int blocks = static_cast<int>(max_rows < 148 * 8 ? max_rows : 148 * 8);
    if (blocks < 1) blocks = 1;
    return launch_kernel(gather_split_kernel, dim3(blocks), dim3(256), 0, st, chained, static_cast<const uint4 *>(x),
                         sorted_rows, offsets, s.E + s.n_shared, s.T, s.k, s.H, max_rows,
                         static_cast<uint2 *>(planes), scale);
}

cudaError_t launch_split_hilo(const moe_shape_t &s, const void *src, int K, const int32_t *offsets,
                              void *planes, float *scale, int64_t max_rows, cudaStream_t st, bool chained,
                              const int32_t *sorted_rows)
{
    int blocks = static_cast<int>(max_rows < 148 * 8 ? max_rows : 148 * 8);
    if (blocks < 1) blocks = 1;
    return launch_kernel(split_hilo_kernel, dim3(blocks), dim3(256), 0, st, chained,
                         static_cast<const uint4 *>(src), K, offsets, s.E + s.n_shared, max_rows,
                         static_cast<uint2 *>(planes), scale, sorted_rows);
}

// ------------------------------------------------------------------ combine
// One block per token; each thread owns 4 consecutive outputs and sums the
// k routed rows (weighted) then the shared rows, in that fixed order.
__global__ void __launch_bounds__(256) combine_kernel(const float4 *__restrict__ y,
                                                      const float *__restrict__ w,
                                                      const int32_t *__restrict__ inv,
                                                      const int32_t *__restrict__ offsets, int H,
                                                      int k, int E, int n_shared, uint2 *out)
{
    grid_dep_wait();
    grid_dep_launch();
    const int t = blockIdx.x;
    const int n4 = H / 4;
    __shared__ int s_slot[kMaxTopK + 1];
    __shared__ float s_w[kMaxTopK];
    if (threadIdx.x < k) {
        s_slot[threadIdx.x] = inv[static_cast<size_t>(t) * k + threadIdx.x];
        s_w[threadIdx.x] = w[static_cast<size_t>(t) * k + threadIdx.x];
    }
    __syncthreads();
    // block (t, y) owns 4-column groups [y*256, (y+1)*256) of token t
    for (int c = blockIdx.y * blockDim.x + threadIdx.x; c < n4; c += gridDim.y * blockDim.x) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j = 0; j < k; ++j) {
            const int slot = s_slot[j];
            if (slot < 0) continue;
            const float wt = s_w[j];
            const float4 v = __ldg(y + static_cast<size_t>(slot) * n4 + c);
            acc.x = fmaf(wt, v.x, acc.x);
            acc.y = fmaf(wt, v.y, acc.y);
            acc.z = fmaf(wt, v.z, acc.z);
            acc.w = fmaf(wt, v.w, acc.w);
        }
        for (int s = 0; s < n_shared; ++s) {
            const float4 v = __ldg(y + static_cast<size_t>(offsets[E + s] + t) * n4 + c);
            acc.x += v.x;
            acc.y += v.y;
            acc.z += v.z;
            acc.w += v.w;
        }
        const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
        const __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
        uint2 o;
        o.x = *reinterpret_cast<const uint32_t *>(&lo);
        o.y = *reinterpret_cast<const uint32_t *>(&hi);
        out[static_cast<size_t>(t) * n4 + c] = o;
    }
}

cudaError_t launch_combine(const moe_shape_t &s, const float *y, const float *w,
                           const int32_t *inv, const int32_t *offsets, void *out, cudaStream_t st,
                           bool chained)
{
    const dim3 grid(s.T, (s.H / 4 + 255) / 256);
    return launch_kernel(combine_kernel, grid, dim3(256), 0, st, chained, reinterpret_cast<const float4 *>(y),
                         w, inv, offsets, s.H, s.k, s.E, s.n_shared, static_cast<uint2 *>(out));
}

}  // namespace moe
