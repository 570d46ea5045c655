// grouped_gemm.cu - persistent grouped expert GEMM on the 5th-generation
// tensor cores (tcgen05 + tensor memory), fed by TMA.
//
// What it computes (the two expert GEMMs of the fused-MoE layer):
//   mode 0:  h_s = SiLU(sc * xp_s . W1[e]^T) * (sc * xp_s . W3[e]^T)
//   mode 1:  y_s = sc * h_s . W2[e]^T
// for every row s of expert e's segment of the permuted activations, with fp32
// accumulation and sc = activation scale * per-expert weight scale.
//
// Operand order ("Swap-AB", from "Mixture-of-Experts kernel engineering on
// Amazon SageMaker AI", abstract, the B^T[N,K] x A^T[K,M] = C^T[N,M] passage,
// and the Russian summary's section "Swap-AB: развернуть матрицы под WGMMA"):
// the tensor core's M extent is fixed (128 rows for a one-CTA tcgen05.mma),
// so when an expert sees few token rows the kernel puts 128 expert-weight rows
// in M and the token rows in N (16..256, chosen per tile at run time).  The
// normal order puts 128 token rows in M and 256 weight rows in N.  Both give
// the same result up to fp32 summation order.
//
// Structure (one CTA per SM, 192 threads):
//   warp 0      TMA producer: weight and activation tiles into a smem ring
//   warp 1      tcgen05.mma issuer (one thread) and tensor-memory owner
//   warps 2..5  epilogue: tcgen05.ld the fp32 accumulator, scale, SwiGLU,
//               convert and store
// Accumulators are double-buffered in tensor memory so the epilogue of one
// tile overlaps the main loop of the next.  Work is split over the grid as
// whole tiles for all full rounds and, for the remaining tiles, as equal
// contiguous ranges of K-steps ("stream-K"); a tile split across CTAs is
// finished by the last CTA to arrive, which sums the fp32 partials in a fixed
// CTA order (deterministic).  The tile list is derived on the device from the
// segment offsets, so token counts are run-time values and nothing is
// recompiled per batch size.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include <mutex>

#include "common.cuh"
#include "ptx.cuh"

namespace moe {

struct GemmParams {
    const int32_t *offsets;
    int E_tot;
    int K;            // reduction length in elements
    int n_feat;       // mode 0: I (hidden features); mode 1: H (outputs)
    int w_rows;       // weight rows per expert: 2I (mode 0) or H (mode 1)
    int out_ld;       // row stride of the output, elements
    void *out;
    const float *wscale;
    float ascale;     // activation scale (1 for bf16 activations)
    float qscale;     // mode 0 with E4M3 output: h is stored as e4m3(h / qscale)
    int32_t *status;
    int32_t *counters;
    float *partials;
    const float *rowscale;   // kHiLo: scale of each permuted activation row
    int lo_rows;             // kHiLo: row offset of the lo plane in the activation map
    int pdl;          // launched as a programmatic dependent: prefetch the first weight
                      // stages into L2 before waiting for the previous kernel
    int rsplit;       // which experts' segments: 0 all; 1 those of 256 rows or more;
                      // 2 the others
    int test_stall;   // test of the abort path only (0 otherwise): in a CTA pair, rank
                      // 1's producer stops after this many stage fills, so that rank
                      // 0's waits run out and the pair's abort tear-down runs
    int wait_at_end;  // the previous kernel is a launch over other experts of the same
                      // GEMM (the CTA-pair launch before an rsplit = 2 launch):
                      // nothing read here depends on it, so wait for it only before
                      // exiting, which keeps dependency waits transitive for the
                      // kernels after this one
    int stream_k;     // 0: whole tiles only.  Otherwise the largest idle share, in
                      // percent of all rounds, that whole tiles may leave: above it the
                      // tiles of the last one or two rounds are split into equal K-step
                      // ranges (stream-K, each tile shared by at most ~2 CTAs).
    int split_cost;   // ... unless the idle whole-tile work per CTA is at most this
                      // many K-steps: the cost of splitting (a split item's epilogue,
                      // partial store and fixup) in main-loop K-steps
    const int32_t *sorted_rows;   // slot -> row code (combine)
    int T, k, R, n_shared;        // tokens, top-k, routed rows T*k, shared experts
    // Fused combine (mode 1): instead of y in slot order, each row is staged
    // as ystage[t][j] (row code f = t*k + j, or shared expert s as j = k + s)
    // and counted per (token, output-feature tile); the CTA that brings a
    // token's count to k + n_shared writes out[t] for that tile's features:
    // sum_j w[t,j] * y[t,j] (fma, in j order) + sum_s y[t,k+s], rounded to
    // bf16 -- the arithmetic and order of the separate combine step.
    int combine;
    float *ystage;
    int32_t *tok_cnt;             // [T][n_ct], zero on entry
    int n_ct;                     // output-feature tiles per token row
    const float *wts;             // router weights [T, k]
    __nv_bfloat16 *comb_out;      // out [T, H]
    // Swap-AB GEMM1 of the layer: once its own loads are issued, the producer
    // prefetches into L2 up to next_prefetch_bytes of the down projection's
    // weights (map tm_next) for the tiles GEMM2 will give this unit first
    long long next_prefetch_bytes;
    int next_K, next_n_feat, next_reverse;
};

template <int kMode, bool kSwap, bool kFp8, int kBN, bool kHiLo = false, bool kPair = false>
struct Cfg {
    // K bytes per operand row and stage: the 128-byte swizzle (64-byte rows
    // with the 64-byte swizzle measured slower for the normal order on B200).
    static constexpr int kRowBytes = 128;
    static constexpr int kMmaPerStage = kRowBytes / 32;     // 32 bytes of K per MMA
    static constexpr int kStageA = 128 * kRowBytes;          // 128 rows
    // kHiLo (E4M3 weights, bf16 activations): each token row arrives as two
    // E4M3 planes (hi, lo), stacked in N: rows [0, n) hi, [n, 2n) lo
    static constexpr int kPlanes = kHiLo ? 2 : 1;
    static constexpr int kStageB = kPlanes * kBN * kRowBytes;
    static constexpr int kStage = kStageA + kStageB;
    static constexpr int kDynBudget = 205 * 1024;
    static constexpr int kStagesRaw = kDynBudget / kStage;
    static constexpr int kStages = kStagesRaw > 12 ? 12 : kStagesRaw;
    // Normal order: kStages stages of kStage bytes.  Swap-AB: the stage size
    // is set per launch from the largest segment (capped at the tile), so a
    // decode batch whose experts see few rows keeps more stages in flight:
    // up to kSlots stages in a ring of kRingBytes.
    static constexpr int kSlots = kSwap ? 12 : kStages;
    static constexpr int kRingBytes = kSwap ? (kDynBudget / 1024) * 1024 : kStages * kStage;
    static constexpr int kDynSmem = kRingBytes + 1024;
    // epilogue warps 2 .. 2+kEpiWarps-1; the normal order uses two per
    // tensor-memory lane quarter, each taking half of the tile's columns
    static constexpr int kEpiWarps = kSwap ? 4 : 8;
    static constexpr int kEpiThreads = 32 * kEpiWarps;
    static constexpr int kThreads = 64 + kEpiThreads;
    static constexpr int kAccCols = kSwap ? kPlanes * kBN : 256;   // fp32 columns per accumulator
    static constexpr int kTmemCols = (2 * kAccCols) <= 32 ? 32 : 2 * kAccCols;
    // token rows per tile (kPair: a CTA pair's tile, 128 rows in each CTA)
    static constexpr int kRowsTile = kSwap ? kBN : (kPair ? 256 : 128);
    static constexpr int kFeatTile = kMode == 0 ? (kSwap ? 64 : 128) : (kSwap ? 128 : 256);
    static constexpr int kKStage = kFp8 ? kRowBytes : kRowBytes / 2;   // K elements per work step
    static constexpr uint32_t kFmt = kFp8 ? 0u : 1u;
    // h leaves GEMM1 as E4M3 only on the all-E4M3 path
    static constexpr bool kOutE4M3 = kFp8 && !kHiLo;
    static_assert(kStages >= 2, "smem ring too small");
    static_assert(!kSwap || kRingBytes >= 2 * kStage, "Swap-AB ring must hold two full-size stages");
    static_assert(!kHiLo || (kSwap && kFp8 && kBN == 16), "hi/lo planes: Swap-AB on the E4M3 tensor path, 16-row tiles");
    // kPair: normal order on a CTA pair (tcgen05 .cta_group::2): M = 256 token
    // rows (128 per CTA), N = 256 weight rows (each CTA stages its 128), each
    // CTA's tensor memory holds its 128 rows x 256 columns
    static_assert(!kPair || (!kSwap && !kHiLo && kBN == 128), "CTA pairs: normal order, 128-row B halves");
    static_assert(kTmemCols <= 512, "tensor memory");
};

// Work item: one tile (expert e, feature tile ft, row tile rt) over K-steps
// [kb, ke).  `partial` is set when the item is one CTA's share of a split tile.
struct Item {
    int e, ft, rt, kb, ke;
    int partial;
    int sk_tile;       // index among stream-K tiles (counters / fixup)
    int slot;          // this CTA's partial slot
};

struct Sched {
    int n_tiles, KT, G, dp_tiles, sk_tiles, sk_ctas;
    int reverse;       // walk the tile list from its end (schedule position t is tile n_tiles-1-t)
    long long sk_total;
};

// Smallest CTA index whose stream-K range contains K-step `i`.
__device__ __forceinline__ int sk_cta_of(long long i, const Sched &S)
{
    return static_cast<int>(((i + 1) * S.sk_ctas + S.sk_total - 1) / S.sk_total) - 1;
}

__device__ __forceinline__ long long sk_begin(int c, const Sched &S)
{
    return static_cast<long long>(c) * S.sk_total / S.sk_ctas;
}

// Iterator over the work items of CTA `c`: first its contiguous K-step range
// of the stream-K region, then whole tiles c, c+G, ... below dp_tiles.  With
// the split items first, the fixup of a split tile (by its last contributor)
// overlaps whole-tile main loops instead of landing in the kernel's tail.
struct ItemIter {
    int c, i_dp;
    long long it, it_end;
    bool in_dp, first_sk;
};

__device__ __forceinline__ void iter_init(ItemIter &I, const Sched &S, int c)
{
    I.c = c;
    I.i_dp = 0;
    I.in_dp = false;
    I.first_sk = true;
    if (c < S.sk_ctas) {
        I.it = sk_begin(c, S);
        I.it_end = sk_begin(c + 1, S);
    } else {
        I.it = I.it_end = 0;
    }
}

template <int kRowsTile, int kFeatTileUnused>
__device__ __forceinline__ void tile_coords(int t, const int *s_prefix, const int *s_lo, const int *s_hi, int Et,
                                            int n_ft, int &e, int &ft, int &rt)
{
    int lo = 0, hi = Et - 1;                 // largest e with prefix[e] <= t
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_prefix[mid] <= t) lo = mid;
        else hi = mid - 1;
    }
    e = lo;
    const int seg = s_hi[e] - s_lo[e];
    const int nrt = (seg + kRowsTile - 1) / kRowsTile;
    const int local = t - s_prefix[e];
    rt = local % nrt;
    ft = local / nrt;
}

template <int kRowsTile>
__device__ __forceinline__ bool iter_next(ItemIter &I, const Sched &S, const int *s_prefix,
                                          const int *s_lo, const int *s_hi, int Et, int n_ft, Item &out)
{
    if (!I.in_dp) {
        if (I.it < I.it_end) {
            const int tl = static_cast<int>(I.it / S.KT);
            const int kb = static_cast<int>(I.it % S.KT);
            const long long left = I.it_end - I.it;
            const int ke = static_cast<int>(left < S.KT - kb ? kb + left : S.KT);
            const int tt = S.dp_tiles + tl;
            tile_coords<kRowsTile, 0>(S.reverse ? S.n_tiles - 1 - tt : tt, s_prefix, s_lo, s_hi, Et, n_ft, out.e,
                                      out.ft, out.rt);
            out.kb = kb;
            out.ke = ke;
            out.partial = !(kb == 0 && ke == S.KT);
            out.sk_tile = tl;
            out.slot = 2 * I.c + (I.first_sk ? 0 : 1);
            I.first_sk = false;
            I.it += ke - kb;
            return true;
        }
        I.in_dp = true;
    }
    const int t = I.c + I.i_dp * S.G;
    if (t >= S.dp_tiles) return false;
    ++I.i_dp;
    tile_coords<kRowsTile, 0>(S.reverse ? S.n_tiles - 1 - t : t, s_prefix, s_lo, s_hi, Et, n_ft, out.e, out.ft,
                              out.rt);
    out.kb = 0;
    out.ke = S.KT;
    out.partial = 0;
    out.sk_tile = -1;
    out.slot = -1;
    return true;
}

// SiLU(g) * u with the hardware exponential and an approximate reciprocal
// (a few ulp of fp32: far below the bf16 / E4M3 rounding of h).  For very
// negative g, 1 + e^-g overflows to +inf and the quotient is -0.
__device__ __forceinline__ float silu_mul(float g, float u)
{
    return __fdividef(g, 1.0f + __expf(-g)) * u;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b)
{
    const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&v);
}

__device__ __forceinline__ uint32_t e4m3_code(float v)
{
    return static_cast<uint32_t>(__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3)) & 0xFFu;
}

// Wait (bounded, ignoring the abort flag) for the last `issued` fills of a
// ring whose next stage/phase is (stage, phase): lets in-flight TMA copies
// land before an aborting CTA exits.
__device__ __forceinline__ void drain_ring(uint64_t *full, int nstages, int stage, uint32_t phase, int issued)
{
    for (int i = 0; i < nstages && i < issued; ++i) {
        stage = stage == 0 ? nstages - 1 : stage - 1;
        if (stage == nstages - 1) phase ^= 1u;
        volatile int no_abort = 0;
        mbar_wait(smem_u32(&full[stage]), phase, &no_abort);
    }
}

template <int kMode, bool kSwap, bool kFp8, int kBN, bool kHiLo = false, bool kPair = false>
__global__ void __launch_bounds__(Cfg<kMode, kSwap, kFp8, kBN, kHiLo, kPair>::kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tm_w,
                        const __grid_constant__ CUtensorMap tm_x,
                        const __grid_constant__ CUtensorMap tm_next, GemmParams p)
{
    using C = Cfg<kMode, kSwap, kFp8, kBN, kHiLo, kPair>;
    extern __shared__ uint8_t dyn_smem[];
    // rows [s_lo[e], s_hi[e]) of expert e's padded segment are this launch's
    // (with p.rsplit, the whole segment or none of it)
    __shared__ int s_lo[kMaxExpertsTotal], s_hi[kMaxExpertsTotal];
    __shared__ int s_prefix[kMaxExpertsTotal + 1];
    __shared__ __align__(8) uint64_t s_full[C::kSlots], s_empty[C::kSlots];
    __shared__ int s_max_seg;
    __shared__ __align__(8) uint64_t s_tfull[2], s_tempty[2], s_drain;
    __shared__ uint32_t s_tmem_base;
    __shared__ volatile int s_abort;
    __shared__ int s_is_last;
    __shared__ int s_slot_of[kMaxCtas];     // stream-K fixup: partial slot of each contributor
    __shared__ float s_xchg[kMode == 0 && kSwap ? 16 * 64 : 1];
    // normal order: per-warp staging of 32 rows x 64 bytes (80-byte pitch, no
    // bank conflicts) so that the output is written as whole row segments
    constexpr int kStagePitch = 80;
    __shared__ __align__(16) uint8_t s_out_stage[kSwap ? 16 : C::kEpiWarps * 32 * kStagePitch];
    // fused combine, per tile: each row's staging row and token, and the
    // tokens this CTA finishes
    constexpr int kTileRowsCta = kSwap ? kBN : 128;
    __shared__ int s_dst[kMode == 1 ? kTileRowsCta : 1];
    __shared__ int s_tok[kMode == 1 ? kTileRowsCta : 1];
    __shared__ int s_fin[kMode == 1 ? kTileRowsCta : 1];
    __shared__ int s_nfin;
    // kPair tear-down: stage fills this CTA's producer issued, and the peer's
    // fill count and abort flag (written by the peer)
    __shared__ int s_fills, s_peer_fills, s_peer_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int Et = p.E_tot;
    // kPair: CTA `rank` of the pair; the pair is one unit of the tile schedule
    const uint32_t rank = kPair ? cluster_ctarank() : 0u;
    const int unit = kPair ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
    uint8_t *tiles = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dyn_smem) + 1023) &
                                                 ~static_cast<uintptr_t>(1023));

    // ---- set-up: barriers, tensor memory, tile table ----
    if (threadIdx.x == 0) {
        s_abort = 0;
        s_fills = 0;
        s_peer_fills = 0;
        s_peer_abort = 0;
        for (int i = 0; i < C::kSlots; ++i) {
            mbar_init(smem_u32(&s_full[i]), 1);
            mbar_init(smem_u32(&s_empty[i]), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(&s_tfull[i]), 1);
            // kPair: rank 0's accumulator barrier also counts the peer's epilogue warps
            mbar_init(smem_u32(&s_tempty[i]), (kPair ? 2 : 1) * C::kEpiWarps);
        }
        mbar_init(smem_u32(&s_drain), 1);
        fence_mbar_init();
        prefetch_tmap(&tm_w);
        prefetch_tmap(&tm_x);
    }
    if (warp == 1) {
        if constexpr (kPair) {
            tmem_alloc_pair(smem_u32(&s_tmem_base), C::kTmemCols);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(smem_u32(&s_tmem_base), C::kTmemCols);
            tmem_relinquish();
        }
    }
    const int n_ft = (p.n_feat + C::kFeatTile - 1) / C::kFeatTile;
    if (warp == 2) {
        // L2 load: under PDL this runs before grid_dep_wait(); the offsets
        // come from the align kernel, which has completed by then
        bool bad = false;
        for (int e = lane; e < Et; e += 32) {
            const int a = __ldcg(p.offsets + e), b = __ldcg(p.offsets + e + 1);
            if (b < a || ((b - a) & 15) != 0 || (a & 15) != 0) bad = true;
            const bool big = b - a >= 256;
            s_lo[e] = a;
            s_hi[e] = p.rsplit == 0 ? b : (p.rsplit == 1 ? (big ? b : a) : (big ? a : b));
        }
        __syncwarp();
        const int per = (Et + 31) / 32;
        const int lo = min(Et, lane * per), hi = min(Et, lo + per);
        int sum = 0, mx = 0;
        for (int e = lo; e < hi; ++e) {
            const int seg = s_hi[e] - s_lo[e];
            mx = max(mx, seg);
            sum += seg > 0 ? ((seg + C::kRowsTile - 1) / C::kRowsTile) * n_ft : 0;
        }
        int inc = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += v;
        }
        int run = inc - sum;
        for (int e = lo; e < hi; ++e) {
            s_prefix[e] = run;
            const int seg = s_hi[e] - s_lo[e];
            run += seg > 0 ? ((seg + C::kRowsTile - 1) / C::kRowsTile) * n_ft : 0;
        }
        if (lane == 31) s_prefix[Et] = inc;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        if (lane == 0) s_max_seg = mx;
        if (__any_sync(0xffffffffu, bad) && lane == 0) {
            set_status(p.status, MOE_ERR_DEVICE_CHECK);
            s_prefix[Et] = 0;   // no work: refuse mis-aligned segments
        }
    }
    tc_fence_before();
    __syncthreads();
    if constexpr (kPair) cluster_sync();   // the peer's barriers exist before any signal crosses
    tc_fence_after();
    const uint32_t tmem_base = s_tmem_base;

    // ring geometry of this launch (Swap-AB: room for the largest tile's rows)
    const int tile_rows_max = max(16, min(C::kRowsTile, s_max_seg));
    const int stage_bytes = kSwap ? C::kStageA + C::kPlanes * tile_rows_max * C::kRowBytes : C::kStage;
    const int n_stages = kSwap ? min(C::kSlots, C::kRingBytes / stage_bytes) : C::kStages;

    Sched S;
    S.n_tiles = s_prefix[Et];
    // A Swap-AB down projection walks its tile list backwards.  With the combine
    // fused, the last expert's tiles would otherwise finish nearly every token
    // (a shared expert, after all the routed ones), piling the finishing work
    // into the kernel's tail; backwards it is spread over the routed experts'
    // tiles.  The standalone call walks the same way, so that both split the
    // same tiles for stream-K and give the same bits.
    S.reverse = kMode == 1 && kSwap ? 1 : 0;
    S.KT = p.K / C::kKStage;
    S.G = kPair ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
    const int rem = S.n_tiles % S.G;
    // whole tiles throughout when the idle share of the last round, over
    // all rounds, is at most p.stream_k percent, or when the idle K-steps
    // per CTA are fewer than a split would cost
    const int rounds = (S.n_tiles + S.G - 1) / S.G;
    const long long idle = static_cast<long long>(S.G) * rounds - S.n_tiles;
    const bool full_enough = S.n_tiles >= S.G && (100 * idle <= static_cast<long long>(p.stream_k) * S.G * rounds ||
                                                  idle * S.KT <= static_cast<long long>(p.split_cost) * S.G);
    if (!p.stream_k || rem == 0) S.dp_tiles = S.n_tiles;
    else if (S.n_tiles < S.G) S.dp_tiles = 0;
    else if (full_enough) S.dp_tiles = S.n_tiles;
    else S.dp_tiles = (S.n_tiles / S.G - 1) * S.G;
    S.sk_tiles = S.n_tiles - S.dp_tiles;
    S.sk_total = static_cast<long long>(S.sk_tiles) * S.KT;
    S.sk_ctas = static_cast<int>(S.sk_total < S.G ? S.sk_total : S.G);

    // ---- programmatic dependent launch ----
    // Everything above reads only the offsets.  The weights are never written
    // by an earlier kernel, so the producer first pulls the opening stages of
    // this CTA's weight stream into L2; every thread then waits for the
    // previous kernel (which wrote the activations this kernel reads) before
    // touching anything else in global memory.
    if (warp == 0 && lane == 0 && p.pdl) {
        constexpr int kHalf = kSwap ? 64 : 128;   // weight rows per gate/up half-tile
        ItemIter I;
        iter_init(I, S, unit);
        Item it;
        int n = 0;
        while (n < n_stages && iter_next<C::kRowsTile>(I, S, s_prefix, s_lo, s_hi, Et, n_ft, it)) {
            const int wbase = it.e * p.w_rows;
            for (int kk = it.kb; kk < it.ke && n < n_stages; ++kk, ++n) {
                const int kx = kk * C::kKStage;
                if (kPair) {
                    // this CTA's half: gate (rank 0) or up (rank 1) rows; W2 rows [128 rank, +128)
                    tma_prefetch_l2_2d(&tm_w, kx, kMode == 0 ? wbase + (rank ? p.n_feat : 0) + it.ft * 128
                                                             : wbase + it.ft * 256 + 128 * static_cast<int>(rank));
                } else if (kMode == 0 && kSwap) {
                    tma_prefetch_l2_4d(&tm_w, kx, it.ft * kHalf, 0, it.e);
                } else if (kMode == 0) {
                    tma_prefetch_l2_2d(&tm_w, kx, wbase + it.ft * kHalf);
                    tma_prefetch_l2_2d(&tm_w, kx, wbase + p.n_feat + it.ft * kHalf);
                } else {
                    tma_prefetch_l2_2d(&tm_w, kx, wbase + it.ft * 2 * kHalf);
                }
            }
        }
    }
    if (!p.wait_at_end) grid_dep_wait();
    grid_dep_launch();


    if (warp == 0) {
        // ================= TMA producer =================
        if (lane == 0) {
            // Swap-AB (few token rows per expert) streams every weight byte
            // once: keep it from displacing the reused activations.  In the
            // normal order a weight tile is reused by all of the expert's row
            // tiles, so it gets the default policy.
            const uint64_t pol_w = kSwap ? policy_evict_first() : policy_evict_normal();
            const uint64_t pol_x = policy_evict_last();
            int stage = 0;
            uint32_t phase = 0;
            int in_flight = 0;
            ItemIter I;
            iter_init(I, S, unit);
            Item it;
            bool ok = true;
            while (ok && iter_next<C::kRowsTile>(I, S, s_prefix, s_lo, s_hi, Et, n_ft, it)) {
                const int row0 = s_lo[it.e] + it.rt * C::kRowsTile;
                const int rows = min(C::kRowsTile, s_hi[it.e] - row0);
                const int wbase = it.e * p.w_rows;
                for (int kk = it.kb; kk < it.ke; ++kk) {
                    if (kPair && p.test_stall > 0 && rank == 1 && in_flight >= p.test_stall) {
                        ok = false;
                        break;
                    }
                    if (!mbar_wait(smem_u32(&s_empty[stage]), phase ^ 1u, &s_abort)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&s_full[stage]);
                    // Swap-AB: only the tile's own token rows (16-row boxes), of
                    // both planes for kHiLo.  kPair: rank 0's barrier counts the
                    // bytes of both CTAs.
                    if (!kPair || rank == 0)
                        mbar_arrive_expect_tx(fb, kSwap ? C::kStageA + C::kPlanes * rows * C::kRowBytes
                                                        : (kPair ? 2 : 1) * C::kStage);
                    const uint32_t sa = smem_u32(tiles + stage * stage_bytes);
                    const uint32_t sb = sa + C::kStageA;
                    const int kx = kk * C::kKStage;
                    if (kSwap) {
                        // one instruction per operand where the layout allows:
                        // the single producer thread's work per stage bounds
                        // the weight stream
                        if (kMode == 0)   // the expert's 64 gate rows, then its 64 up rows (4-D map)
                            tma_load_4d(sa, &tm_w, fb, kx, it.ft * 64, 0, it.e, pol_w);
                        else
                            tma_load_2d(sa, &tm_w, fb, kx, wbase + it.ft * 128, pol_w);
                        if (kHiLo)        // 16 token rows of the hi plane, then of the lo plane (3-D map)
                            tma_load_3d(sb, &tm_x, fb, kx, row0, 0, pol_x);
                        else
                            for (int rr = 0; rr < rows; rr += 16)
                                tma_load_2d(sb + rr * C::kRowBytes, &tm_x, fb, kx, row0 + rr, pol_x);
                    } else if (kPair) {
                        // this CTA's 128 token rows and its half of the 256 weight
                        // rows (gate or up rows of 128 features; W2 rows [128 rank, +128))
                        const uint32_t fb0 = mapa_shared(fb, 0);
                        tma_load_2d_pair(sa, &tm_x, fb0, kx, row0 + 128 * static_cast<int>(rank), pol_x);
                        tma_load_2d_pair(sb, &tm_w, fb0, kx,
                                         kMode == 0 ? wbase + (rank ? p.n_feat : 0) + it.ft * 128
                                                    : wbase + it.ft * 256 + 128 * static_cast<int>(rank),
                                         pol_w);
                    } else {
                        tma_load_2d(sa, &tm_x, fb, kx, row0, pol_x);
                        if (kMode == 0) {
                            tma_load_2d(sb, &tm_w, fb, kx, wbase + it.ft * 128, pol_w);
                            tma_load_2d(sb + 128 * C::kRowBytes, &tm_w, fb, kx, wbase + p.n_feat + it.ft * 128, pol_w);
                        } else {
                            tma_load_2d(sb, &tm_w, fb, kx, wbase + it.ft * 256, pol_w);
                        }
                    }
                    ++in_flight;
                    if (++stage == n_stages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if constexpr (kMode == 0 && kSwap) {
                if (ok && p.next_prefetch_bytes > 0) {
                    // GEMM2's tile list is GEMM1's with n_ft2 feature tiles of 128
                    // rows instead of n_ft (the same row tiles per expert)
                    const int n_ft2 = (p.next_n_feat + 127) / 128;
                    const int n_tiles2 = s_prefix[Et] / n_ft * n_ft2;
                    const int KT2 = p.next_K / C::kKStage;
                    long long budget = p.next_prefetch_bytes;
                    for (int ts = unit; ts < n_tiles2 && budget > 0; ts += S.G) {
                        const int t = p.next_reverse ? n_tiles2 - 1 - ts : ts;   // GEMM2's walk order
                        int lo = 0, hi = Et - 1;
                        while (lo < hi) {
                            const int mid = (lo + hi + 1) >> 1;
                            if (s_prefix[mid] / n_ft * n_ft2 <= t) lo = mid;
                            else hi = mid - 1;
                        }
                        const int seg = s_hi[lo] - s_lo[lo];
                        const int nrt = (seg + C::kRowsTile - 1) / C::kRowsTile;
                        const int ft2 = (t - s_prefix[lo] / n_ft * n_ft2) / nrt;
                        const int wrow = lo * p.next_n_feat + ft2 * 128;
                        for (int kk = 0; kk < KT2 && budget > 0; ++kk, budget -= 128 * C::kRowBytes)
                            tma_prefetch_l2_2d(&tm_next, kk * C::kKStage, wrow);
                    }
                }
            }
            s_fills = in_flight;
            if (!ok) {
                // let issued copies land (kPair: rank 1's copies complete on rank
                // 0's barriers; the pair retires its fills at tear-down)
                if (!kPair) drain_ring(s_full, n_stages, stage, phase, in_flight);
            } else if (kPair) {
                // every stage this CTA filled has been consumed, so no commit of
                // rank 0's MMAs is still on its way to this CTA's barriers
                drain_ring(s_empty, n_stages, stage, phase, in_flight);
            }
        }
    } else if (warp == 1) {
        // ================= MMA issuer (kPair: rank 0 only) =================
        if (lane == 0 && (!kPair || rank == 0)) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            ItemIter I;
            iter_init(I, S, unit);
            Item it;
            bool ok = true;
            // kPair: both barriers below also receive the peer CTA's arrivals
            auto wait_bar = [&](uint32_t bar, uint32_t parity) -> bool {
                return kPair ? mbar_wait_cluster(bar, parity, &s_abort) : mbar_wait(bar, parity, &s_abort);
            };
            while (ok && iter_next<C::kRowsTile>(I, S, s_prefix, s_lo, s_hi, Et, n_ft, it)) {
                if (!wait_bar(smem_u32(&s_tempty[acc]), acc_phase ^ 1u)) break;
                tc_fence_after();
                const uint32_t d = tmem_base + acc * C::kAccCols;
                int n = 256;
                if (kSwap) {
                    const int seg = s_hi[it.e] - s_lo[it.e];
                    n = C::kPlanes * min(C::kRowsTile, seg - it.rt * C::kRowsTile);
                }
                const uint32_t idesc = idesc_make(C::kFmt, kPair ? 256 : 128, n);
                for (int kk = it.kb; kk < it.ke; ++kk) {
                    if (!wait_bar(smem_u32(&s_full[stage]), phase)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(tiles + stage * stage_bytes);
                    const uint32_t sb = sa + C::kStageA;
#pragma unroll
                    for (int s = 0; s < C::kMmaPerStage; ++s) {
                        const uint64_t ad = sdesc_k_sw128(sa + s * 32);
                        const uint64_t bd = sdesc_k_sw128(sb + s * 32);
                        const uint32_t accum = (kk > it.kb || s > 0) ? 1u : 0u;
                        if constexpr (kPair) {
                            if (kFp8) mma_e4m3_pair(d, ad, bd, idesc, accum);
                            else mma_bf16_pair(d, ad, bd, idesc, accum);
                        } else {
                            if (kFp8) mma_e4m3(d, ad, bd, idesc, accum);
                            else mma_bf16(d, ad, bd, idesc, accum);
                        }
                    }
                    // kPair: the stage is free in both CTAs
                    if constexpr (kPair) mma_commit_pair(smem_u32(&s_empty[stage]), 3);
                    else mma_commit(smem_u32(&s_empty[stage]));
                    if (++stage == n_stages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                if constexpr (kPair) mma_commit_pair(smem_u32(&s_tfull[acc]), 3);   // both epilogues
                else mma_commit(smem_u32(&s_tfull[acc]));
                if (++acc == 2) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
            // every MMA issued above has completed once this barrier fires
            if constexpr (kPair) mma_commit_pair(smem_u32(&s_drain), 1);
            else mma_commit(smem_u32(&s_drain));
            volatile int no_abort = 0;
            mbar_wait(smem_u32(&s_drain), 0, &no_abort);
        }
    } else if (warp >= 2 && warp < 2 + C::kEpiWarps) {
        // ================= epilogue (warps 2 .. 2+kEpiWarps-1) ==============
        const int q = warp & 3;                 // tensor-memory lane quarter
        const int r = q * 32 + lane;            // accumulator row of this thread
        const int etid = threadIdx.x - 64;      // 0 .. kEpiThreads-1
        const int ch = (warp - 2) >> 2;         // column half (normal order, 8 warps)
        constexpr int kNch = C::kEpiWarps / 4;  // column halves
        int acc = 0;
        uint32_t acc_phase = 0;
        ItemIter I;
        iter_init(I, S, unit);
        Item it;
        while (iter_next<C::kRowsTile>(I, S, s_prefix, s_lo, s_hi, Et, n_ft, it)) {
            const bool got = kPair ? mbar_wait_cluster(smem_u32(&s_tfull[acc]), acc_phase, &s_abort)
                                   : mbar_wait(smem_u32(&s_tfull[acc]), acc_phase, &s_abort);
            if (!named_bar_and(1, C::kEpiThreads, got)) break;   // all epilogue warps agree
            tc_fence_after();
            const int seg = s_hi[it.e] - s_lo[it.e];
            // kPair: this CTA holds rows [128 rank, 128 rank + 128) of the pair's tile
            const int row0 = s_lo[it.e] + it.rt * C::kRowsTile + (kPair ? 128 * static_cast<int>(rank) : 0);
            const int rows = kPair ? max(0, min(128, seg - it.rt * C::kRowsTile - 128 * static_cast<int>(rank)))
                                   : min(C::kRowsTile, seg - it.rt * C::kRowsTile);
            // output scale of the tile; kHiLo: times the activation row's own
            // scale (column j of a Swap-AB tile is permuted row row0 + j)
            const float sc = (kHiLo ? 1.0f : p.ascale) * (p.wscale ? __ldg(&p.wscale[it.e]) : 1.0f);
            // fused combine: each row's staging row and token (-1 for pad
            // slots), a per-tile table filled by all epilogue threads before use
            if constexpr (kMode == 1 && kSwap) {
                for (int i = etid; p.combine && i < rows; i += C::kEpiThreads) {
                    const int code = __ldg(p.sorted_rows + row0 + i);
                    int t = -1, dst = -1;
                    if (code >= 0) {
                        const int kS = p.k + p.n_shared;
                        if (code < p.R) {
                            t = code / p.k;
                            dst = t * kS + (code - t * p.k);
                        } else {
                            const int sh = (code - p.R) / p.T;
                            t = code - p.R - sh * p.T;
                            dst = t * kS + p.k + sh;
                        }
                    }
                    s_dst[i] = dst;
                    s_tok[i] = t;
                }
                if (p.combine) {
                    if (etid == 0) s_nfin = 0;
                    named_bar_sync(1, C::kEpiThreads);
                }
            }
            // kHiLo: times the activation row's own scale (column j of a
            // Swap-AB tile is permuted row row0 + j)
            auto col_sc = [&](int j) -> float { return kHiLo ? sc * __ldg(&p.rowscale[row0 + j]) : sc; };
            // Fused combine, after this CTA has staged its rows of the tile:
            // count each row in for (token, feature tile) and finish the tokens
            // whose last row this was (output features [h0, h0 + fcols)).
            // The staging stores of all epilogue threads are ordered before each
            // arrival by the barrier and the arriving thread's fence; the
            // finishing CTA's fence after its arrival orders its reads after
            // every other CTA's stores.  The finishing work is spread over all
            // epilogue threads as (token, 4 features) items, kU items per thread
            // at a time with all their loads issued before any is used.
            auto combine_tail = [&](int nrows, int h0, int fcols) {
                named_bar_sync(1, C::kEpiThreads);
                const int kS = p.k + p.n_shared;
                for (int i = etid; i < nrows; i += C::kEpiThreads) {
                    const int t = s_tok[i];
                    if (t < 0) continue;
                    __threadfence();
                    if (atomicAdd(&p.tok_cnt[static_cast<size_t>(t) * p.n_ct + it.ft], 1) == kS - 1)
                        s_fin[atomicAdd(&s_nfin, 1)] = t;
                }
                named_bar_sync(1, C::kEpiThreads);
                const int nf = s_nfin;
                if (nf == 0) return;
                __threadfence();
                const int ngrp = min(fcols, p.n_feat - h0) / 4;      // 4-feature groups
                const int items = nf * ngrp;
                // rows of a token prefetched per item (the rest load in order) and
                // items per thread at a time
                constexpr int kU = 2;
                constexpr int kMaxS = 9;
                for (int base = etid; base < items; base += kU * C::kEpiThreads) {
                    float4 v[kU][kMaxS];
                    int tk[kU], g4[kU];
#pragma unroll
                    for (int u = 0; u < kU; ++u) {
                        const int item = base + u * C::kEpiThreads;
                        tk[u] = item < items ? s_fin[item / ngrp] : -1;
                        g4[u] = item < items ? item % ngrp : 0;
                        if (tk[u] < 0) continue;
                        const float4 *yr = reinterpret_cast<const float4 *>(
                            p.ystage + static_cast<size_t>(tk[u]) * kS * p.out_ld + h0 + 4 * g4[u]);
#pragma unroll
                        for (int j = 0; j < kMaxS; ++j)
                            if (j < kS) v[u][j] = __ldcg(yr + static_cast<size_t>(j) * (p.out_ld / 4));
                    }
#pragma unroll
                    for (int u = 0; u < kU; ++u) {
                        if (tk[u] < 0) continue;
                        const float4 *yr = reinterpret_cast<const float4 *>(
                            p.ystage + static_cast<size_t>(tk[u]) * kS * p.out_ld + h0 + 4 * g4[u]);
                        const float *wt = p.wts + static_cast<size_t>(tk[u]) * p.k;
                        float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
                        // sum_j w_j y_j (fma, j order), then the shared rows
                        auto add_row = [&](int j, const float4 &y) {
                            if (j < p.k) {
                                const float wj = __ldg(wt + j);
                                a.x = fmaf(wj, y.x, a.x);
                                a.y = fmaf(wj, y.y, a.y);
                                a.z = fmaf(wj, y.z, a.z);
                                a.w = fmaf(wj, y.w, a.w);
                            } else {
                                a.x += y.x;
                                a.y += y.y;
                                a.z += y.z;
                                a.w += y.w;
                            }
                        };
#pragma unroll
                        for (int j = 0; j < kMaxS; ++j)
                            if (j < kS) add_row(j, v[u][j]);
                        for (int j = kMaxS; j < kS; ++j) add_row(j, __ldcg(yr + static_cast<size_t>(j) * (p.out_ld / 4)));
                        *reinterpret_cast<uint2 *>(p.comb_out + static_cast<size_t>(tk[u]) * p.out_ld + h0 + 4 * g4[u]) =
                            make_uint2(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w));
                    }
                }
            };
            const uint32_t tacc = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * C::kAccCols;
            // 16 accumulator columns starting at c0 (kHiLo: hi plane + lo plane)
            auto ld_acc16 = [&](int c0, uint32_t (&v)[16]) {
                tmem_ld16(tacc + c0, v);
                if constexpr (kHiLo) {
                    uint32_t w2[16];
                    tmem_ld16(tacc + rows + c0, w2);
                    tmem_wait_ld();
#pragma unroll
                    for (int i2 = 0; i2 < 16; ++i2) v[i2] = __float_as_uint(__uint_as_float(v[i2]) + __uint_as_float(w2[i2]));
                }
            };
            const int ncols = kSwap ? rows : 256;
            if (!it.partial) {
                if (kSwap && kMode == 0) {
                    // rows 0..63 gate, 64..127 up for features f0 .. f0+63
                    const int f0 = it.ft * 64;
                    for (int c0 = 0; c0 < ncols; c0 += 16) {
                        uint32_t v[16];
                        ld_acc16(c0, v);
                        tmem_wait_ld();
                        if (q >= 2)
#pragma unroll
                            for (int j = 0; j < 16; ++j) s_xchg[j * 64 + (r - 64)] = __uint_as_float(v[j]);
                        named_bar_sync(1, 128);
                        if (q < 2) {
#pragma unroll
                            for (int j = 0; j < 16; ++j) {
                                const float scj = col_sc(c0 + j);
                                const float g = __uint_as_float(v[j]) * scj;
                                const float u = s_xchg[j * 64 + r] * scj;
                                const float hv = silu_mul(g, u);
                                const size_t o = static_cast<size_t>(row0 + c0 + j) * p.out_ld + f0 + r;
                                if (C::kOutE4M3)
                                    static_cast<uint8_t *>(p.out)[o] = static_cast<uint8_t>(e4m3_code(hv / p.qscale));
                                else
                                    static_cast<__nv_bfloat16 *>(p.out)[o] = __float2bfloat16_rn(hv);
                            }
                        }
                        named_bar_sync(1, 128);
                    }
                } else if (kSwap) {
                    const int h0 = it.ft * 128;
                    for (int c0 = 0; c0 < ncols; c0 += 16) {
                        uint32_t v[16];
                        ld_acc16(c0, v);
                        tmem_wait_ld();
                        if (p.combine) {
#pragma unroll
                            for (int j = 0; j < 16; ++j) {
                                const int dr = s_dst[c0 + j];
                                if (dr >= 0)
                                    p.ystage[static_cast<size_t>(dr) * p.out_ld + h0 + r] = __uint_as_float(v[j]) * col_sc(c0 + j);
                            }
                        } else {
#pragma unroll
                            for (int j = 0; j < 16; ++j)
                                static_cast<float *>(p.out)[static_cast<size_t>(row0 + c0 + j) * p.out_ld + h0 + r] =
                                    __uint_as_float(v[j]) * col_sc(c0 + j);
                        }
                    }
                } else if (kMode == 0) {
                    // 32 features per chunk: h row segment of 64 (bf16) or 32 (E4M3) bytes
                    const int f0 = it.ft * 128;
                    uint8_t *stg = s_out_stage + (warp - 2) * 32 * kStagePitch;
                    const float inv_q = C::kOutE4M3 ? 1.0f / p.qscale : 1.0f;
                    for (int c0 = ch * (128 / kNch); c0 < (ch + 1) * (128 / kNch); c0 += 32) {
                        uint32_t g[16], u[16], g2[16], u2[16];
                        tmem_ld16(tacc + c0, g);
                        tmem_ld16(tacc + 128 + c0, u);
                        tmem_ld16(tacc + c0 + 16, g2);
                        tmem_ld16(tacc + 128 + c0 + 16, u2);
                        tmem_wait_ld();
                        float hv[32];
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            hv[j] = silu_mul(__uint_as_float(g[j]) * sc, __uint_as_float(u[j]) * sc);
                            hv[16 + j] = silu_mul(__uint_as_float(g2[j]) * sc, __uint_as_float(u2[j]) * sc);
                        }
                        uint4 *wr = reinterpret_cast<uint4 *>(stg + lane * kStagePitch);
                        if (C::kOutE4M3) {
#pragma unroll
                            for (int j = 0; j < 2; ++j) {
                                uint32_t w4[4];
#pragma unroll
                                for (int i2 = 0; i2 < 4; ++i2) {
                                    const int b = 16 * j + 4 * i2;
                                    w4[i2] = e4m3_code(hv[b] * inv_q) | (e4m3_code(hv[b + 1] * inv_q) << 8) |
                                             (e4m3_code(hv[b + 2] * inv_q) << 16) | (e4m3_code(hv[b + 3] * inv_q) << 24);
                                }
                                wr[j] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                            }
                        } else {
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                wr[j] = make_uint4(pack_bf16x2(hv[8 * j], hv[8 * j + 1]), pack_bf16x2(hv[8 * j + 2], hv[8 * j + 3]),
                                                   pack_bf16x2(hv[8 * j + 4], hv[8 * j + 5]), pack_bf16x2(hv[8 * j + 6], hv[8 * j + 7]));
                        }
                        __syncwarp();
                        constexpr int kSegLanes = C::kOutE4M3 ? 2 : 4;          // 16-byte pieces per row segment
                        constexpr int kRowsPerPass = 32 / kSegLanes;
                        const size_t esz = C::kOutE4M3 ? 1 : 2;
#pragma unroll
                        for (int ps = 0; ps < kSegLanes; ++ps) {
                            const int rl = ps * kRowsPerPass + lane / kSegLanes;
                            const int rg = q * 32 + rl;
                            const uint4 val = *reinterpret_cast<const uint4 *>(stg + rl * kStagePitch + (lane % kSegLanes) * 16);
                            if (rg < rows)
                                *reinterpret_cast<uint4 *>(static_cast<uint8_t *>(p.out) +
                                                           (static_cast<size_t>(row0 + rg) * p.out_ld + f0 + c0) * esz +
                                                           (lane % kSegLanes) * 16) = val;
                        }
                        __syncwarp();
                    }
                } else {
                    // 16 fp32 columns per chunk: y row segment of 64 bytes
                    const int h0 = it.ft * 256;
                    uint8_t *stg = s_out_stage + (warp - 2) * 32 * kStagePitch;
                    for (int c0 = ch * (256 / kNch); c0 < (ch + 1) * (256 / kNch); c0 += 16) {
                        if (h0 + c0 >= p.n_feat) break;
                        uint32_t v[16];
                        ld_acc16(c0, v);
                        tmem_wait_ld();
                        float4 *wr = reinterpret_cast<float4 *>(stg + lane * kStagePitch);
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            wr[j] = make_float4(__uint_as_float(v[4 * j]) * sc, __uint_as_float(v[4 * j + 1]) * sc,
                                                __uint_as_float(v[4 * j + 2]) * sc, __uint_as_float(v[4 * j + 3]) * sc);
                        __syncwarp();
#pragma unroll
                        for (int ps = 0; ps < 4; ++ps) {
                            const int rl = ps * 8 + (lane >> 2);
                            const int rg = q * 32 + rl;
                            const float4 val = *reinterpret_cast<const float4 *>(stg + rl * kStagePitch + (lane & 3) * 16);
                            if (rg < rows)
                                *reinterpret_cast<float4 *>(static_cast<float *>(p.out) +
                                                            static_cast<size_t>(row0 + rg) * p.out_ld + h0 + c0 + (lane & 3) * 4) = val;
                        }
                        __syncwarp();
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    // kPair: the accumulator is free once both CTAs' epilogues are done
                    if constexpr (kPair) mbar_arrive_cluster(mapa_shared(smem_u32(&s_tempty[acc]), 0));
                    else mbar_arrive(smem_u32(&s_tempty[acc]));
                }
                if constexpr (kMode == 1 && kSwap)
                    if (p.combine) combine_tail(rows, it.ft * 128, 128);
            } else if constexpr (kSwap) {
                // ---- one share of a split tile: store the raw partial ----
                // (decode only: prefill launches take whole tiles)
                float *slot = p.partials + static_cast<size_t>(it.slot) * 128 * C::kAccCols;
                for (int c0 = ch * (ncols / kNch); c0 < (ch + 1) * (ncols / kNch); c0 += 16) {
                    uint32_t v[16];
                    ld_acc16(c0, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 16; ++j) __stcg(&slot[(c0 + j) * 128 + r], __uint_as_float(v[j]));
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&s_tempty[acc]));
                __threadfence();
                named_bar_sync(1, C::kEpiThreads);
                // contributing CTAs of this tile, in K order
                const long long t_it0 = static_cast<long long>(it.sk_tile) * S.KT;
                const int c_first = sk_cta_of(t_it0, S);
                const int c_last = sk_cta_of(t_it0 + S.KT - 1, S);
                if (etid == 0) {
                    const int old = atomicAdd(&p.counters[it.sk_tile], 1);
                    s_is_last = (old == c_last - c_first);
                }
                named_bar_sync(1, C::kEpiThreads);
                if (s_is_last) {
                    __threadfence();
                    // partial slot of every contributing CTA, once (64-bit divisions)
                    for (int c = c_first + etid; c <= c_last; c += C::kEpiThreads) {
                        const int first_tile = static_cast<int>(sk_begin(c, S) / S.KT);
                        s_slot_of[c - c_first] = 2 * c + (first_tile == it.sk_tile ? 0 : 1);
                    }
                    named_bar_sync(1, C::kEpiThreads);
                    auto slot_of = [&](int c) -> const float * {
                        return p.partials + static_cast<size_t>(s_slot_of[c - c_first]) * 128 * C::kAccCols;
                    };
                    if (kSwap && kMode == 0) {
                        const int f0 = it.ft * 64;
                        const int rr = etid & 63;
                        for (int j = etid >> 6; j < ncols; j += 2) {
                            float g = 0.f, u = 0.f;
                            for (int c = c_first; c <= c_last; ++c) {
                                const float *ps = slot_of(c);
                                g += __ldcg(&ps[j * 128 + rr]);
                                u += __ldcg(&ps[j * 128 + 64 + rr]);
                            }
                            const float scj = col_sc(j);
                            const float hv = silu_mul(g * scj, u * scj);
                            const size_t o = static_cast<size_t>(row0 + j) * p.out_ld + f0 + rr;
                            if (C::kOutE4M3) static_cast<uint8_t *>(p.out)[o] = static_cast<uint8_t>(e4m3_code(hv / p.qscale));
                            else static_cast<__nv_bfloat16 *>(p.out)[o] = __float2bfloat16_rn(hv);
                        }
                    } else if (kSwap) {
                        const int h0 = it.ft * 128;
                        for (int j = 0; j < ncols; ++j) {
                            float a = 0.f;
                            for (int c = c_first; c <= c_last; ++c) a += __ldcg(&slot_of(c)[j * 128 + etid]);
                            if (!p.combine)
                                static_cast<float *>(p.out)[static_cast<size_t>(row0 + j) * p.out_ld + h0 + etid] = a * col_sc(j);
                            else if (s_dst[j] >= 0)
                                p.ystage[static_cast<size_t>(s_dst[j]) * p.out_ld + h0 + etid] = a * col_sc(j);
                        }
                        if constexpr (kMode == 1)
                            if (p.combine) combine_tail(ncols, h0, 128);
                    }
                }
                named_bar_sync(1, C::kEpiThreads);
            }
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
    }

    // ---- tear-down ----
    tc_fence_before();
    __syncthreads();
    if constexpr (kPair) {
        // Each CTA tells the other how many stage fills it issued and whether
        // it aborted; neither leaves while the other may still signal it.
        if (threadIdx.x == 0) {
            st_shared_cluster(mapa_shared(smem_u32(&s_peer_fills), rank ^ 1u), static_cast<uint32_t>(s_fills));
            st_shared_cluster(mapa_shared(smem_u32(&s_peer_abort), rank ^ 1u), static_cast<uint32_t>(s_abort));
        }
        cluster_sync();
        if (s_abort || s_peer_abort) {                  // the same decision in both CTAs
            // After an abort some copies may still be landing.  Both CTAs' halves
            // of fill i complete on rank 0's full barrier of stage i % n_stages,
            // in phase (i / n_stages) & 1.  Rank 0 retires the last ring's worth
            // of fills: a fill only rank 1 issued is armed for its half, a fill
            // only rank 0 issued gets rank 1's half counted as done, then every
            // phase is awaited (bounded), so no copy into either CTA is in flight
            // when they leave.  Older fills were consumed by the MMAs already.
            if (rank == 0 && threadIdx.x == 0) {
                const int n0 = s_fills, n1 = s_peer_fills, nmax = max(n0, n1);
                for (int i = max(0, nmax - n_stages); i < nmax; ++i) {
                    const uint32_t fb = smem_u32(&s_full[i % n_stages]);
                    if (i >= n0) mbar_arrive_expect_tx(fb, C::kStage);
                    else if (i >= n1) mbar_complete_tx(fb, C::kStage);
                    volatile int no_abort = 0;
                    mbar_wait(fb, static_cast<uint32_t>((i / n_stages) & 1), &no_abort);
                }
            }
            cluster_sync();
        }
    }
    if (threadIdx.x == 0 && s_abort) set_status(p.status, MOE_ERR_TIMEOUT);
    if (warp == 1) {
        tc_fence_after();
        if constexpr (kPair) tmem_dealloc_pair(tmem_base, C::kTmemCols);
        else tmem_dealloc(tmem_base, C::kTmemCols);
    }
    if (p.wait_at_end) grid_dep_wait();
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// Map over a row-major tensor of 2 to 4 dimensions (dims[0] the contiguous
// one) with the 128-byte swizzle; a box is 128 bytes of dims[0] times box[1..]
// of the others.  A map depends only on these arguments (not on the device
// or on what the memory holds), so the last few are kept per host thread and
// a repeat call with the same buffers skips the encode.
static bool make_map_nd(CUtensorMap *m, const void *base, bool u8, int rank, const uint64_t *dims,
                        const uint32_t *box)
{
    // dims[0] = cols (elements, contiguous), dims[1..] row-major outer extents;
    // box[0] is implied (128 bytes of cols)
    struct Entry {
        const void *base;
        int rank;
        uint64_t dims[4];
        uint32_t box[4];
        bool u8, valid;
        CUtensorMap map;
    };
    constexpr int kEntries = 16;
    thread_local Entry cache[kEntries] = {};
    thread_local int next = 0;
    for (int i = 0; i < kEntries; ++i) {
        const Entry &c = cache[i];
        bool same = c.valid && c.base == base && c.rank == rank && c.u8 == u8;
        for (int d = 0; same && d < rank; ++d) same = c.dims[d] == dims[d] && (d == 0 || c.box[d] == box[d]);
        if (same) {
            *m = c.map;
            return true;
        }
    }
    constexpr uint32_t row_bytes = 128;
    EncodeTiledFn fn = get_encode_fn();
    if (!fn) return false;
    const uint32_t esz = u8 ? 1 : 2;
    cuuint64_t gdims[4], strides[3];
    cuuint32_t gbox[4], estr[4] = {1, 1, 1, 1};
    uint64_t pitch = dims[0] * esz;
    for (int d = 0; d < rank; ++d) {
        gdims[d] = dims[d];
        gbox[d] = d == 0 ? row_bytes / esz : box[d];
        if (d > 0) {
            strides[d - 1] = pitch;
            pitch *= dims[d];
        }
    }
    CUresult r = fn(m, u8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                    static_cast<cuuint32_t>(rank), const_cast<void *>(base), gdims, strides, gbox, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return false;
    Entry &c = cache[next];
    next = (next + 1) % kEntries;
    c = Entry{base, rank, {0, 0, 0, 0}, {0, 0, 0, 0}, u8, true, *m};
    for (int d = 0; d < rank; ++d) {
        c.dims[d] = dims[d];
        c.box[d] = box[d];
    }
    return true;
}

// 2-D map over a row-major [rows, cols] matrix with 128-byte rows per box
// and the 128-byte swizzle; box = box_rows x (128 bytes).
static bool make_map(CUtensorMap *m, const void *base, bool u8, uint64_t rows, uint64_t cols, uint32_t box_rows)
{
    const uint64_t dims[2] = {cols, rows};
    const uint32_t box[2] = {0, box_rows};
    return make_map_nd(m, base, u8, 2, dims, box);
}

// SMs of the current device (the persistent grid size), cached per device.
static int sm_count()
{
    static std::atomic<int> cache[64];
    int dev = 0;
    cudaGetDevice(&dev);
    int n = (dev >= 0 && dev < 64) ? cache[dev].load(std::memory_order_relaxed) : 0;
    if (n == 0) {
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 148;
        if (n > kMaxCtas) n = kMaxCtas;
        if (dev >= 0 && dev < 64) cache[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

// Persistent grid of CTA pairs for a kPair kernel on the current device: as
// many pairs as can be resident at once (two SMs of one GPC each), at most
// half the SM count.  Cached per kernel configuration and device.
template <class Cf, typename Kern>
static int pair_grid(Kern kern)
{
    static std::atomic<int> cache[64];
    int dev = 0;
    cudaGetDevice(&dev);
    int grid = (dev >= 0 && dev < 64) ? cache[dev].load(std::memory_order_relaxed) : 0;
    if (grid == 0) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * (sm_count() / 2));
        cfg.blockDim = dim3(Cf::kThreads);
        cfg.dynamicSmemBytes = Cf::kDynSmem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int clusters = 0;
        if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) != cudaSuccess || clusters <= 0) {
            cudaGetLastError();
            clusters = 1;
        }
        grid = 2 * (clusters < sm_count() / 2 ? clusters : sm_count() / 2);
        if (dev >= 0 && dev < 64) cache[dev].store(grid, std::memory_order_relaxed);
    }
    return grid;
}

template <int kMode, bool kSwap, bool kFp8, int kBN, bool kHiLo = false, bool kPair = false>
static cudaError_t run_gemm(const moe_shape_t &s, const GemmArgs &a, cudaStream_t st, int *host_err)
{
    using Cf = Cfg<kMode, kSwap, kFp8, kBN, kHiLo, kPair>;
    auto kern = grouped_gemm_kernel<kMode, kSwap, kFp8, kBN, kHiLo, kPair>;
    static PerDeviceOnce attrs;          // function attributes are per device
    attrs([&] { cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cf::kDynSmem); });
    const int Et = s.E + s.n_shared;
    const bool u8 = kFp8;              // activations are E4M3 codes
    const bool u8w = kFp8;             // weights are E4M3 codes
    const int K = kMode == 0 ? s.H : s.I;
    const uint64_t w_rows = kMode == 0 ? 2ull * s.I : static_cast<uint64_t>(s.H);
    // weight box rows: Swap-AB gate/up halves (64) or W2 rows (128); normal
    // gate/up halves (128) or W2 rows (256); a CTA of a pair: 128
    const uint32_t wbox = kSwap ? (kMode == 0 ? 64 : 128) : (kMode == 0 || kPair ? 128 : 256);
    const uint32_t xbox = kSwap ? 16 : 128;     // Swap-AB loads token rows in 16-row boxes
    CUtensorMap tm_w, tm_x, tm_next;
    static_assert(Cf::kRowBytes == 128, "tensor maps use 128-byte rows with the 128-byte swizzle");
    // Swap-AB gate/up: [Et][2][I][H] as 4-D, one box = an expert's 64 gate
    // rows and 64 up rows; hi/lo activations: [2][max_rows][K] as 3-D, one
    // box = 16 rows of both planes
    const uint64_t wdims[4] = {static_cast<uint64_t>(K), static_cast<uint64_t>(s.I), 2, static_cast<uint64_t>(Et)};
    const uint32_t wbox4[4] = {0, 64, 2, 1};
    const uint64_t xdims[3] = {static_cast<uint64_t>(K), static_cast<uint64_t>(a.max_rows), 2};
    const uint32_t xbox3[3] = {0, 16, 2};
    const bool w_ok = kSwap && kMode == 0 ? make_map_nd(&tm_w, a.wgt, u8w, 4, wdims, wbox4)
                                          : make_map(&tm_w, a.wgt, u8w, Et * w_rows, K, wbox);
    const bool x_ok = kHiLo ? make_map_nd(&tm_x, a.act, u8, 3, xdims, xbox3)
                            : make_map(&tm_x, a.act, u8, Cf::kPlanes * a.max_rows, K, xbox);
    if (!w_ok || !x_ok) {
        *host_err = MOE_ERR_CUDA;
        return cudaSuccess;
    }
    // the down projection's weights [Et * H, I], 128-row boxes, for the L2
    // prefetch at the end of a Swap-AB GEMM1 (else an unused copy of tm_w)
    const bool prefetch_next = kMode == 0 && kSwap && a.next_wgt != nullptr;
    if (prefetch_next) {
        if (!make_map(&tm_next, a.next_wgt, u8w, static_cast<uint64_t>(Et) * s.H, s.I, 128)) {
            *host_err = MOE_ERR_CUDA;
            return cudaSuccess;
        }
    } else {
        tm_next = tm_w;
    }
    GemmParams p{};
    p.offsets = a.offsets;
    p.E_tot = Et;
    p.K = K;
    p.n_feat = kMode == 0 ? s.I : s.H;
    p.w_rows = static_cast<int>(w_rows);
    p.out_ld = kMode == 0 ? s.I : s.H;
    p.out = a.out;
    p.wscale = a.wscale;
    p.ascale = a.ascale;
    p.qscale = a.qscale;
    p.status = a.status;
    p.counters = a.counters;
    p.partials = a.partials;
    p.rowscale = a.rowscale;
    p.lo_rows = static_cast<int>(a.max_rows);
    p.sorted_rows = a.sorted_rows;
    p.T = s.T;
    p.k = s.k;
    p.R = s.T * s.k;
    p.n_shared = s.n_shared;
    p.combine = kMode == 1 && kSwap && a.combine ? 1 : 0;   // the combine is fused on the Swap-AB path only
    p.ystage = a.ystage;
    p.tok_cnt = a.tok_cnt;
    p.n_ct = (s.H + (kSwap ? 127 : 255)) / (kSwap ? 128 : 256);
    p.wts = a.wts;
    p.comb_out = static_cast<__nv_bfloat16 *>(a.comb_out);
    p.next_prefetch_bytes = prefetch_next ? a.next_prefetch_bytes : 0;
    p.next_K = s.I;
    p.next_n_feat = s.H;
    p.next_reverse = a.next_reverse ? 1 : 0;
    p.rsplit = a.rsplit;
    p.wait_at_end = a.wait_at_end ? 1 : 0;
    p.test_stall = kPair ? a.test_stall : 0;
    // When to split tiles.  Decode (Swap-AB): above 3% idle, unless the idle
    // work is under 12 K-steps per CTA.  A split item's epilogue (partial
    // store, fixup, combine) costs about that much of the weight stream: on
    // the DeepSeek-V3 down projection for one token (504 tiles of 16 K-steps
    // on 148 SMs, 15% idle) whole tiles measured 7% faster than splitting,
    // while long-K tiles (Mixtral, 224 K-steps) gain from splitting.  Prefill
    // (normal order) takes whole tiles: a split tile carries 128 KB of fp32
    // partials, and splitting the one-CTA launch over the segments' last rows
    // made the Qwen2 and Mixtral down projections 35-40% slower.
    p.stream_k = kSwap ? 3 : 0;
    p.split_cost = kSwap ? 12 : 0;
    p.pdl = a.chained ? 1 : 0;
    if (!a.chained) {
        cudaError_t err = cudaMemsetAsync(a.counters, 0, 2 * kMaxCtas * sizeof(int32_t), st);
        if (err != cudaSuccess) return err;
    }
    if constexpr (kPair) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(pair_grid<Cf>(kern));
        cfg.blockDim = dim3(Cf::kThreads);
        cfg.dynamicSmemBytes = Cf::kDynSmem;
        cfg.stream = st;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = a.chained ? 2 : 1;
        return cudaLaunchKernelEx(&cfg, kern, tm_w, tm_x, tm_next, p);
    } else {
        return launch_kernel(kern, dim3(sm_count()), dim3(Cf::kThreads), Cf::kDynSmem, st, a.chained, tm_w, tm_x,
                             tm_next, p);
    }
}

cudaError_t launch_grouped_gemm(const moe_shape_t &s, const GemmPlan &p, const GemmArgs &a,
                                cudaStream_t st, int *launches, int *host_err)
{
    *host_err = MOE_OK;
    const bool fp8 = s.adtype == MOE_E4M3;
    const bool w8 = s.wdtype == MOE_E4M3 && s.adtype == MOE_BF16;
    cudaError_t err = cudaSuccess;
    if (w8) {
        // E4M3 weights with bf16 activations: the activation rows are first
        // split into two E4M3 planes under a per-row power-of-two scale
        // (v = s * (hi + lo)), then the grouped GEMM runs on the E4M3 tensor
        // path with both planes stacked in N.
        if (!a.chained) {
            err = cudaMemsetAsync(a.counters, 0, 2 * kMaxCtas * sizeof(int32_t), st);
            if (err != cudaSuccess) return err;
        }
        GemmArgs g = a;
        if (!(a.mode == 0 && a.planes_ready)) {
            err = launch_split_hilo(s, a.act, a.mode == 0 ? s.H : s.I, a.offsets, a.planes, a.rowscale,
                                    a.max_rows, st, a.chained, a.skip_pad_rows);
            if (err != cudaSuccess) return err;
            *launches += 1;
            g.chained = true;      // counters are zero; a dependent launch of the split
        }
        g.act = a.planes;
#define MOE_W8(MODE, BN) err = run_gemm<MODE, true, true, BN, true>(s, g, st, host_err)
        // hi/lo tiles take 16 token rows (plan_gemm)
        if (a.mode == 0) MOE_W8(0, 16);
        else MOE_W8(1, 16);
#undef MOE_W8
        *launches += 1;
        return err;
    }
#define MOE_G(MODE, SWAP, FP8, BN) err = run_gemm<MODE, SWAP, FP8, BN>(s, a, st, host_err)
#define MOE_BY_BN(MODE, FP8)                      \
    switch (p.bn) {                               \
    case 16: MOE_G(MODE, true, FP8, 16); break;   \
    case 32: MOE_G(MODE, true, FP8, 32); break;   \
    case 64: MOE_G(MODE, true, FP8, 64); break;   \
    case 128: MOE_G(MODE, true, FP8, 128); break; \
    default: MOE_G(MODE, true, FP8, 256); break;  \
    }
    if (p.swap) {
        if (a.mode == 0) {
            if (fp8) { MOE_BY_BN(0, true) } else { MOE_BY_BN(0, false) }
        } else {
            if (fp8) { MOE_BY_BN(1, true) } else { MOE_BY_BN(1, false) }
        }
    } else {
        // Normal order (prefill).  Experts with 256 rows or more run on CTA
        // pairs (256 x 256 tiles, half the weight bytes staged per SM), the
        // others on one-CTA 128-row tiles in a second launch, which pads at
        // most 127 rows per expert where a pair tile pads up to 255.  Each
        // expert's weights are read by one launch only (splitting a segment
        // between the two launches read its weights twice from HBM).  The
        // second launch reads nothing the first writes: it starts as the
        // pairs' SMs free up and waits for them only before exiting.
        GemmArgs g = a;
        g.rsplit = 1;
        if (a.mode == 0) {
            if (fp8) err = run_gemm<0, false, true, 128, false, true>(s, g, st, host_err);
            else err = run_gemm<0, false, false, 128, false, true>(s, g, st, host_err);
        } else {
            if (fp8) err = run_gemm<1, false, true, 128, false, true>(s, g, st, host_err);
            else err = run_gemm<1, false, false, 128, false, true>(s, g, st, host_err);
        }
        if (err != cudaSuccess || *host_err != MOE_OK) return err;
        *launches += 1;
        g.test_stall = 0;
        g.rsplit = 2;
        g.chained = true;
        g.wait_at_end = true;
        if (a.mode == 0) {
            if (fp8) err = run_gemm<0, false, true, 256>(s, g, st, host_err);
            else err = run_gemm<0, false, false, 256>(s, g, st, host_err);
        } else {
            if (fp8) err = run_gemm<1, false, true, 256>(s, g, st, host_err);
            else err = run_gemm<1, false, false, 256>(s, g, st, host_err);
        }
    }
#undef MOE_BY_BN
#undef MOE_G
    *launches += 1;
    return err;
}

}  // namespace moe
