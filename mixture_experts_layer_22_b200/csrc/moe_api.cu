// moe_api.cu - the extern "C" boundary of libmoe_b200.so (declared in
// include/moe.h): argument validation, workspace carving and the launch
// sequence of the fused layer.  No call allocates device memory, reads device
// data on the host (except moe_get_device_status) or synchronises.
#include <cstdio>
#include <cstring>

#include "common.cuh"

namespace moe {

static thread_local int g_launches = 0;

int &launch_counter() { return g_launches; }

static size_t up256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

int validate_shape(const moe_shape_t *s, bool need_gemm)
{
    if (!s) return MOE_ERR_INVALID_ARG;
    if (s->T < 1 || s->H < 1 || s->I < 1 || s->E < 1 || s->k < 1) return MOE_ERR_INVALID_ARG;
    if (s->E > kMaxExperts || s->k > s->E || s->k > kMaxTopK) return MOE_ERR_INVALID_ARG;
    if (s->n_shared < 0 || s->n_shared > 1) return MOE_ERR_INVALID_ARG;
    if (s->gate != MOE_GATE_SOFTMAX && s->gate != MOE_GATE_SIGMOID) return MOE_ERR_INVALID_ARG;
    if (s->wdtype != MOE_BF16 && s->wdtype != MOE_E4M3) return MOE_ERR_INVALID_ARG;
    if (s->adtype != MOE_BF16 && s->adtype != MOE_E4M3) return MOE_ERR_INVALID_ARG;
    if (s->adtype == MOE_E4M3 && s->wdtype != MOE_E4M3) return MOE_ERR_INVALID_ARG;
    if (s->variant < MOE_VARIANT_AUTO || s->variant > MOE_VARIANT_NORMAL) return MOE_ERR_INVALID_ARG;
    if (s->pad < 1 || s->pad > 4096) return MOE_ERR_INVALID_ARG;
    if (static_cast<int64_t>(s->T) * s->k > (1 << 24)) return MOE_ERR_INVALID_ARG;
    if (s->H % 8 != 0) return MOE_ERR_INVALID_ARG;
    if (need_gemm) {
        if (s->H % 128 != 0 || s->I % 128 != 0) return MOE_ERR_UNSUPPORTED;
        if (s->pad % 16 != 0 || s->pad > 256) return MOE_ERR_UNSUPPORTED;
    }
    return MOE_OK;
}

GemmPlan plan_gemm(const moe_shape_t &s)
{
    GemmPlan p;
    // One tcgen05.mma on one SM has a fixed 128-row M extent: when no expert
    // can receive 128 rows or more, weights go to M and tokens to N.
    // E4M3 weights with bf16 activations stack the hi and lo E4M3 planes of
    // the activation rows in the MMA's N, so that path is always Swap-AB.
    p.swap = s.variant == MOE_VARIANT_SWAP_AB || (s.variant == MOE_VARIANT_AUTO && s.T <= 128) ||
             (s.wdtype == MOE_E4M3 && s.adtype == MOE_BF16);
    if (p.swap) {
        const int rows = (s.T + s.pad - 1) / s.pad * s.pad;   // worst case rows of one expert
        int bn = 16;
        // The hi/lo path holds two planes per token row in every stage, and
        // the smem ring is sized per launch from the largest segment (the
        // shared expert's T rows).  Its weight stream is bound by how many
        // bytes each SM keeps in flight, so its tiles take 16 rows: 20 KB
        // stages, 10 in the ring, where 64-row tiles (32 KB stages) kept 6
        // for every expert because of the shared one (measured 3-4% faster at
        // T = 32..128).  The price is that a segment of more than 16 rows
        // takes several row tiles over the same weight tile; those are
        // adjacent in the tile list, so they run at the same time and the
        // repeat reads come from L2.
        const int cap = (s.wdtype == MOE_E4M3 && s.adtype == MOE_BF16) ? 16 : 256;
        while (bn < rows && bn < cap) bn <<= 1;
        p.bn = bn;
    } else {
        p.bn = 256;
    }
    return p;
}

bool ws_layout(const moe_shape_t &s, WsLayout &L)
{
    const int64_t R = static_cast<int64_t>(s.T) * s.k;
    const int Et = s.E + s.n_shared;
    L.max_rows = R + static_cast<int64_t>(s.n_shared) * s.T + static_cast<int64_t>(Et) * (s.pad - 1);
    L.n_chunks = static_cast<int>((R + kAlignChunk - 1) / kAlignChunk);
    const GemmPlan p = plan_gemm(s);
    const bool w8 = s.wdtype == MOE_E4M3 && s.adtype == MOE_BF16;
    L.acc_cols = p.swap ? (w8 ? 2 : 1) * p.bn : 256;
    const size_t ab = s.adtype == MOE_E4M3 ? 1 : 2;
    size_t o = 0;
    L.ctrl = o;        o += up256(sizeof(Ctrl));
    // stream-K tile counters right after the control words (one memset
    // clears both): GEMM1 uses the first half, GEMM2 the second
    L.counters = o;    o += up256(4 * kMaxCtas * 4);
    // the fused combine's arrival counters per (token, 128-feature tile), then
    // the router tickets: all cleared together with the control words
    L.tok_cnt = o;     o += up256(static_cast<size_t>(s.T) * ((s.H + 127) / 128) * 4);
    L.tickets = o;     o += up256(static_cast<size_t>(s.T) * 4);
    L.logits = o;      o += up256(static_cast<size_t>(s.T) * s.E * 4);
    L.ids = o;         o += up256(R * 4);
    L.w = o;           o += up256(R * 4);
    L.counts = o;      o += up256(Et * 4);
    L.offsets = o;     o += up256((Et + 1) * 4);
    L.chunk_hist = o;  o += up256(static_cast<size_t>(L.n_chunks) * Et * 4);
    L.chunk_base = o;  o += up256(static_cast<size_t>(L.n_chunks) * Et * 4);
    L.sorted_rows = o; o += up256(L.max_rows * 4);
    L.inv = o;         o += up256(R * 4);
    L.xp = o;          o += up256(L.max_rows * s.H * ab);
    L.h = o;           o += up256(L.max_rows * s.I * ab);
    // the down projection's rows: in slot order [max_rows, H] fp32 when the
    // combine is its own pass, or staged per (token, choice) [T, k+S, H] when
    // it is fused into the GEMM (at most max_rows rows either way)
    L.y = o;           o += up256(L.max_rows * s.H * 4);
    L.partials = o;    o += up256(static_cast<size_t>(2 * kMaxCtas) * 128 * L.acc_cols * 4);
    // hi/lo E4M3 planes of GEMM1's then GEMM2's activations (reused: the
    // split of h runs after GEMM1 has finished reading the planes of xp)
    const int64_t kmax = s.H > s.I ? s.H : s.I;
    L.planes = o;      o += w8 ? up256(2 * L.max_rows * kmax) : 0;
    L.rowscale = o;    o += w8 ? up256(L.max_rows * 4) : 0;
    L.total = o;
    return true;
}

static bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace moe

using namespace moe;

extern "C" {

int moe_max_rows(const moe_shape_t *shape, int64_t *rows)
{
    int st = validate_shape(shape, false);
    if (st != MOE_OK) return st;
    if (!rows) return MOE_ERR_INVALID_ARG;
    WsLayout L;
    ws_layout(*shape, L);
    *rows = L.max_rows;
    return MOE_OK;
}

int moe_workspace_size(const moe_shape_t *shape, size_t *bytes)
{
    int st = validate_shape(shape, false);
    if (st != MOE_OK) return st;
    if (!bytes) return MOE_ERR_INVALID_ARG;
    WsLayout L;
    ws_layout(*shape, L);
    *bytes = L.total;
    return MOE_OK;
}

int moe_last_launch_count(void) { return g_launches; }

const char *moe_status_string(int status)
{
    switch (status) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape or dtype combination";
    case MOE_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA runtime or driver error";
    case MOE_ERR_DEVICE_CHECK: return "a kernel found invalid data (expert id out of range or mis-aligned segment)";
    case MOE_ERR_TIMEOUT: return "a kernel pipeline wait timed out";
    default: return "unknown status";
    }
}

static int cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

int moe_route_topk(const moe_shape_t *shape, const float *logits, int32_t *ids, float *w,
                   moe_stream_t stream)
{
    g_launches = 0;
    int st = validate_shape(shape, false);
    if (st != MOE_OK) return st;
    if (!logits || !ids || !w) return MOE_ERR_INVALID_ARG;
    g_launches = 1;
    return cuda_status(launch_route(*shape, logits, ids, w, reinterpret_cast<cudaStream_t>(stream)));
}

int moe_align_permute(const moe_shape_t *shape, const int32_t *ids, int32_t *counts,
                      int32_t *offsets, int32_t *sorted_rows, int32_t *inv, void *ws,
                      size_t ws_bytes, moe_stream_t stream)
{
    g_launches = 0;
    int st = validate_shape(shape, false);
    if (st != MOE_OK) return st;
    if (!ids || !counts || !offsets || !sorted_rows || !inv || !ws) return MOE_ERR_INVALID_ARG;
    if (!aligned(ws, 256)) return MOE_ERR_INVALID_ARG;
    WsLayout L;
    ws_layout(*shape, L);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    char *b = static_cast<char *>(ws);
    return cuda_status(launch_align(*shape, ids, counts, offsets, sorted_rows, inv,
                                    reinterpret_cast<int32_t *>(b + L.chunk_hist),
                                    reinterpret_cast<int32_t *>(b + L.chunk_base),
                                    reinterpret_cast<Ctrl *>(b + L.ctrl),
                                    reinterpret_cast<cudaStream_t>(stream), &g_launches));
}

int moe_gather(const moe_shape_t *shape, const void *x, const int32_t *sorted_rows,
               const int32_t *offsets, float a1_scale, void *xp, moe_stream_t stream)
{
    g_launches = 0;
    int st = validate_shape(shape, false);
    if (st != MOE_OK) return st;
    if (!x || !sorted_rows || !offsets || !xp) return MOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(xp, 16)) return MOE_ERR_INVALID_ARG;
    if (shape->adtype == MOE_E4M3 && !(a1_scale > 0.0f)) return MOE_ERR_INVALID_ARG;
    WsLayout L;
    ws_layout(*shape, L);
    g_launches = 1;
    return cuda_status(launch_gather(*shape, x, sorted_rows, offsets, a1_scale, xp, L.max_rows,
                                     reinterpret_cast<cudaStream_t>(stream)));
}

static int gemm_common(const moe_shape_t *shape, int mode, const void *act, const void *wgt,
                       const float *wscale, float ascale, float qscale, const int32_t *offsets,
                       void *out, void *ws, size_t ws_bytes, cudaStream_t stream, int test_stall = 0)
{
    int st = validate_shape(shape, true);
    if (st != MOE_OK) return st;
    if (!act || !wgt || !offsets || !out || !ws) return MOE_ERR_INVALID_ARG;
    if (!aligned(act, 16) || !aligned(wgt, 16) || !aligned(out, 16) || !aligned(ws, 256))
        return MOE_ERR_INVALID_ARG;
    if (shape->wdtype == MOE_E4M3 && !wscale) return MOE_ERR_INVALID_ARG;
    if (shape->adtype == MOE_E4M3 && (!(ascale > 0.0f) || !(qscale > 0.0f))) return MOE_ERR_INVALID_ARG;
    WsLayout L;
    ws_layout(*shape, L);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    char *b = static_cast<char *>(ws);
    GemmArgs a;
    a.chained = false;
    a.mode = mode;
    a.act = act;
    a.wgt = wgt;
    a.wscale = wscale;
    a.ascale = shape->adtype == MOE_E4M3 ? ascale : 1.0f;
    a.qscale = qscale;
    a.offsets = offsets;
    a.out = out;
    a.status = &reinterpret_cast<Ctrl *>(b + L.ctrl)->status;
    a.counters = reinterpret_cast<int32_t *>(b + L.counters);
    a.partials = reinterpret_cast<float *>(b + L.partials);
    a.planes = b + L.planes;
    a.rowscale = reinterpret_cast<float *>(b + L.rowscale);
    a.max_rows = L.max_rows;
    a.test_stall = test_stall;
    int host_err = MOE_OK;
    cudaError_t e = launch_grouped_gemm(*shape, plan_gemm(*shape), a, stream, &g_launches, &host_err);
    if (host_err != MOE_OK) return host_err;
    return cuda_status(e);
}

int moe_grouped_gemm_swiglu(const moe_shape_t *shape, const void *xp, const void *w13,
                            const float *w13_scale, float a1_scale, float a2_scale,
                            const int32_t *offsets, void *h, void *ws, size_t ws_bytes,
                            moe_stream_t stream)
{
    g_launches = 0;
    return gemm_common(shape, 0, xp, w13, w13_scale, a1_scale, a2_scale, offsets, h, ws, ws_bytes,
                       reinterpret_cast<cudaStream_t>(stream));
}

int moe_grouped_gemm_down(const moe_shape_t *shape, const void *h, const void *w2,
                          const float *w2_scale, float a2_scale, const int32_t *offsets, float *y,
                          void *ws, size_t ws_bytes, moe_stream_t stream)
{
    g_launches = 0;
    return gemm_common(shape, 1, h, w2, w2_scale, a2_scale, a2_scale, offsets, y, ws, ws_bytes,
                       reinterpret_cast<cudaStream_t>(stream));
}

int moe_selftest_pair_abort(const moe_shape_t *shape, const void *h, const void *w2, const int32_t *offsets,
                            float *y, void *ws, size_t ws_bytes, moe_stream_t stream)
{
    g_launches = 0;
    if (!shape || plan_gemm(*shape).swap || shape->wdtype != MOE_BF16 || shape->adtype != MOE_BF16)
        return MOE_ERR_UNSUPPORTED;
    return gemm_common(shape, 1, h, w2, nullptr, 1.0f, 1.0f, offsets, y, ws, ws_bytes,
                       reinterpret_cast<cudaStream_t>(stream), 2);
}

int moe_combine(const moe_shape_t *shape, const float *y, const float *w, const int32_t *inv,
                const int32_t *offsets, void *out, moe_stream_t stream)
{
    g_launches = 0;
    int st = validate_shape(shape, false);
    if (st != MOE_OK) return st;
    if (!y || !w || !inv || !offsets || !out) return MOE_ERR_INVALID_ARG;
    if (!aligned(y, 16) || !aligned(out, 8) || shape->H % 4 != 0) return MOE_ERR_INVALID_ARG;
    g_launches = 1;
    return cuda_status(launch_combine(*shape, y, w, inv, offsets, out, reinterpret_cast<cudaStream_t>(stream)));
}

int moe_router_topk(const moe_shape_t *shape, const void *x, const void *wg, float *logits, int32_t *ids,
                    float *w, void *ws, size_t ws_bytes, moe_stream_t stream)
{
    g_launches = 0;
    int st = validate_shape(shape, false);
    if (st != MOE_OK) return st;
    if (!x || !wg || !logits || !ids || !w || !ws) return MOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(wg, 16) || !aligned(ws, 256)) return MOE_ERR_INVALID_ARG;
    WsLayout L;
    ws_layout(*shape, L);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t sm = reinterpret_cast<cudaStream_t>(stream);
    int32_t *tickets = reinterpret_cast<int32_t *>(static_cast<char *>(ws) + L.tickets);
    if (cudaMemsetAsync(tickets, 0, static_cast<size_t>(shape->T) * sizeof(int32_t), sm) != cudaSuccess)
        return MOE_ERR_CUDA;
    g_launches = 1;
    return cuda_status(launch_router(*shape, x, wg, logits, tickets, ids, w, sm, false));
}

// The fused layer from router logits (wg == NULL) or from the router weight.
static int fused_impl(const moe_shape_t *shape, const void *x, const float *logits, const void *wg,
                      const void *w13, const float *w13_scale, const void *w2,
                      const float *w2_scale, float a1_scale, float a2_scale, void *out, void *ws,
                      size_t ws_bytes, moe_stream_t stream)
{
    g_launches = 0;
    int st = validate_shape(shape, true);
    if (st != MOE_OK) return st;
    if (!x || (!logits && !wg) || !w13 || !w2 || !out || !ws) return MOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(out, 16) || !aligned(w13, 16) || !aligned(w2, 16) || !aligned(ws, 256))
        return MOE_ERR_INVALID_ARG;
    if (wg && !aligned(wg, 16)) return MOE_ERR_INVALID_ARG;
    if (shape->wdtype == MOE_E4M3 && (!w13_scale || !w2_scale)) return MOE_ERR_INVALID_ARG;
    if (shape->adtype == MOE_E4M3 && (!(a1_scale > 0.0f) || !(a2_scale > 0.0f))) return MOE_ERR_INVALID_ARG;
    const moe_shape_t &s = *shape;
    WsLayout L;
    ws_layout(s, L);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t sm = reinterpret_cast<cudaStream_t>(stream);
    char *b = static_cast<char *>(ws);
    Ctrl *ctrl = reinterpret_cast<Ctrl *>(b + L.ctrl);
    int32_t *ids = reinterpret_cast<int32_t *>(b + L.ids);
    float *w = reinterpret_cast<float *>(b + L.w);
    int32_t *counts = reinterpret_cast<int32_t *>(b + L.counts);
    int32_t *offsets = reinterpret_cast<int32_t *>(b + L.offsets);
    int32_t *rows = reinterpret_cast<int32_t *>(b + L.sorted_rows);
    int32_t *inv = reinterpret_cast<int32_t *>(b + L.inv);
    void *xp = b + L.xp;
    void *h = b + L.h;
    float *y = reinterpret_cast<float *>(b + L.y);

    cudaError_t e;
    const int n_zero = static_cast<int>((L.tickets - L.ctrl) / sizeof(int32_t));
    if (!wg && s.T <= 32 && static_cast<int64_t>(s.T) * s.k <= kAlignChunk) {
        // A small decode batch (a warp per token): routing and alignment in one block, which first
        // clears the status, the align ticket and both GEMMs' tile counters
        // (adjacent at the start of the workspace).  It is a programmatic
        // dependent launch like every kernel after it: it waits for whatever
        // ran before it on the stream before touching the workspace.
        e = launch_route_align(s, logits, w, counts, offsets, rows, inv, ctrl, reinterpret_cast<int32_t *>(ctrl),
                               n_zero, sm, true);
        if (e != cudaSuccess) return MOE_ERR_CUDA;
        g_launches += 1;
    } else {
        if (wg) {
            // the router kernel counts per-token tickets: one memset clears
            // them with the control words and counters (adjacent)
            e = cudaMemsetAsync(ctrl, 0, L.tickets + static_cast<size_t>(s.T) * sizeof(int32_t) - L.ctrl, sm);
            if (e != cudaSuccess) return MOE_ERR_CUDA;
            e = launch_router(s, x, wg, reinterpret_cast<float *>(b + L.logits),
                              reinterpret_cast<int32_t *>(b + L.tickets), ids, w, sm, false);
        } else {
            // the route kernel (a warp per token) clears the control words and
            // counters itself; like every kernel after it, it is a programmatic
            // dependent launch that waits for the stream's earlier work first
            e = launch_route(s, logits, ids, w, sm, reinterpret_cast<int32_t *>(ctrl), n_zero, true);
        }
        if (e != cudaSuccess) return MOE_ERR_CUDA;
        g_launches += 1;
        e = launch_align(s, ids, counts, offsets, rows, inv, reinterpret_cast<int32_t *>(b + L.chunk_hist),
                         reinterpret_cast<int32_t *>(b + L.chunk_base), ctrl, sm, &g_launches, true);
        if (e != cudaSuccess) return MOE_ERR_CUDA;
    }
    // the gather (E4M3 weights with bf16 activations: gather and hi/lo split
    // in one pass, straight into the planes GEMM1 reads)
    const bool w8 = s.wdtype == MOE_E4M3 && s.adtype == MOE_BF16;
    if (w8)
        e = launch_gather_split(s, x, rows, offsets, b + L.planes, reinterpret_cast<float *>(b + L.rowscale),
                                L.max_rows, sm, true);
    else
        e = launch_gather(s, x, rows, offsets, a1_scale, xp, L.max_rows, sm, true, true);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    g_launches += 1;
    const GemmPlan plan = plan_gemm(s);
    GemmArgs a;
    a.chained = true;
    a.status = &ctrl->status;
    a.counters = reinterpret_cast<int32_t *>(b + L.counters);
    a.partials = reinterpret_cast<float *>(b + L.partials);
    a.planes = b + L.planes;
    a.rowscale = reinterpret_cast<float *>(b + L.rowscale);
    a.max_rows = L.max_rows;
    a.offsets = offsets;
    a.skip_pad_rows = rows;
    int host_err = MOE_OK;
    a.mode = 0;
    a.act = xp;
    a.planes_ready = w8;
    // decode: GEMM1 prefetches the start of GEMM2's weight stream into L2 as
    // it finishes, so that the down projection starts on cached weights
    a.next_wgt = w2;
    a.next_prefetch_bytes = 512 * 1024;
    a.next_reverse = plan.swap;            // GEMM2 fuses the combine (below) and then walks backwards
    a.wgt = w13;
    a.wscale = w13_scale;
    a.ascale = s.adtype == MOE_E4M3 ? a1_scale : 1.0f;
    a.qscale = a2_scale;
    a.out = h;
    e = launch_grouped_gemm(s, plan, a, sm, &g_launches, &host_err);
    if (host_err != MOE_OK) return host_err;
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    // GEMM2.  Decode (Swap-AB): the combine is fused into its epilogue, which
    // writes out; the combine's staging and counting overlap the weight
    // stream and a launch disappears.  Prefill (CTA pairs): the combine is its
    // own pass after GEMM2 -- measured faster there, because the epilogue of a
    // compute-bound 256-row tile has no room for the combine's L2 reads.
    const bool fuse_combine = plan.swap;
    a.mode = 1;
    a.planes_ready = false;
    a.next_wgt = nullptr;
    a.next_prefetch_bytes = 0;
    a.act = h;
    a.wgt = w2;
    a.wscale = w2_scale;
    a.ascale = s.adtype == MOE_E4M3 ? a2_scale : 1.0f;
    a.out = y;
    a.combine = fuse_combine;
    a.sorted_rows = rows;
    a.ystage = y;
    a.tok_cnt = reinterpret_cast<int32_t *>(b + L.tok_cnt);
    a.wts = w;
    a.comb_out = out;
    a.counters += 2 * kMaxCtas;
    e = launch_grouped_gemm(s, plan, a, sm, &g_launches, &host_err);
    if (host_err != MOE_OK) return host_err;
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    if (!fuse_combine) {
        e = launch_combine(s, y, w, inv, offsets, out, sm, true);
        if (e != cudaSuccess) return MOE_ERR_CUDA;
        g_launches += 1;
    }
    return MOE_OK;
}

int moe_fused_forward(const moe_shape_t *shape, const void *x, const float *logits,
                      const void *w13, const float *w13_scale, const void *w2,
                      const float *w2_scale, float a1_scale, float a2_scale, void *out, void *ws,
                      size_t ws_bytes, moe_stream_t stream)
{
    if (!logits) {
        g_launches = 0;
        return MOE_ERR_INVALID_ARG;
    }
    return fused_impl(shape, x, logits, nullptr, w13, w13_scale, w2, w2_scale, a1_scale, a2_scale, out, ws,
                      ws_bytes, stream);
}

int moe_fused_forward_router(const moe_shape_t *shape, const void *x, const void *wg, const void *w13,
                             const float *w13_scale, const void *w2, const float *w2_scale, float a1_scale,
                             float a2_scale, void *out, void *ws, size_t ws_bytes, moe_stream_t stream)
{
    if (!wg) {
        g_launches = 0;
        return MOE_ERR_INVALID_ARG;
    }
    return fused_impl(shape, x, nullptr, wg, w13, w13_scale, w2, w2_scale, a1_scale, a2_scale, out, ws,
                      ws_bytes, stream);
}

int moe_get_device_status(const void *ws, int32_t *status, moe_stream_t stream)
{
    if (!ws || !status) return MOE_ERR_INVALID_ARG;
    cudaStream_t sm = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(sm) != cudaSuccess) return MOE_ERR_CUDA;
    int32_t v = 0;
    if (cudaMemcpy(&v, ws, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
    *status = v;
    return MOE_OK;
}

int moe_reset_device_status(void *ws, moe_stream_t stream)
{
    if (!ws) return MOE_ERR_INVALID_ARG;
    return cuda_status(cudaMemsetAsync(ws, 0, sizeof(int32_t), reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
