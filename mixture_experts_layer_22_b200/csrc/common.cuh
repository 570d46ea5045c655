// common.cuh - internal declarations shared by the library's translation units.
#pragma once
#include <atomic>
#include <cstddef>
#include <cstdint>
#include <mutex>
#include <cuda_runtime.h>

#include "moe.h"

namespace moe {

constexpr int kMaxExperts = 512;            // routed experts per layer
constexpr int kMaxExpertsTotal = kMaxExperts + 1;
constexpr int kMaxTopK = 32;
constexpr int kMaxCtas = 160;               // persistent GEMM grid bound (>= SM count)
constexpr int kAlignChunk = 1024;           // routed rows per align block

// Host-side setup that CUDA keeps per device (function attributes,
// occupancy): runs f once for each device it is called on, thread-safe.
class PerDeviceOnce {
  public:
    template <class F>
    void operator()(F &&f)
    {
        int d = 0;
        cudaGetDevice(&d);
        if (d < 0 || d >= kDevices) {            // beyond the table: always run (idempotent)
            std::lock_guard<std::mutex> g(m_);
            f();
            return;
        }
        if (done_[d].load(std::memory_order_acquire)) return;
        std::lock_guard<std::mutex> g(m_);
        if (!done_[d].load(std::memory_order_relaxed)) {
            f();
            done_[d].store(true, std::memory_order_release);
        }
    }

  private:
    static constexpr int kDevices = 64;
    std::atomic<bool> done_[kDevices]{};
    std::mutex m_;
};

// Control words at the start of the workspace.
struct Ctrl {
    int32_t status;       // first device-side error (moe_status), 0 = none
    int32_t ticket;       // align: blocks finished counting
    int32_t pad_[62];
};

__device__ __forceinline__ void set_status(int32_t *status, int32_t code)
{
    atomicCAS(status, 0, code);
}

// Programmatic dependent launch.  Inside moe_fused_forward each kernel after
// the first is launched while its predecessor still runs.  Every kernel calls
// grid_dep_wait() (the predecessor grid has completed and its writes are
// visible) before it writes anything (other than an atomic first-error
// status) and before it reads what its predecessor writes; only then does it let its own successor launch.  So
// when a kernel starts, every kernel two or more places before it has
// completed: the grouped GEMMs read the segment offsets (written by align)
// and prefetch weights before they wait.  Both calls are no-ops in a kernel
// launched without the attribute.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Every kernel of the library prefers the largest shared-memory carveout: the
// grouped GEMMs need it, and a small kernel that asked for a different split
// of the SM's L1 and shared memory would make the SM switch configuration
// between the launches of one layer call.  Set once per kernel and device.
inline void prefer_max_smem(const void *kern)
{
    static std::mutex m;
    static const void *done_kern[256];
    static int done_dev[256];
    static int n_done = 0;
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> g(m);
    for (int i = 0; i < n_done; ++i)
        if (done_kern[i] == kern && done_dev[i] == dev) return;
    cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    cudaGetLastError();                          // a refusal only leaves the default carveout
    if (n_done < 256) {
        done_kern[n_done] = kern;
        done_dev[n_done] = dev;
        ++n_done;
    }
}

// Launch with the programmatic-stream-serialisation attribute when `pdl`.
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                          bool pdl, Args... args)
{
    prefer_max_smem(reinterpret_cast<const void *>(kern));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// Workspace carving (host side), every region 256-byte aligned.
struct WsLayout {
    size_t ctrl, ids, w, counts, offsets, chunk_hist, chunk_base, sorted_rows, inv;
    size_t xp, h, y, counters, partials;
    size_t tickets, logits;   // router: per-token tickets (zeroed with the control words), logits
    size_t total;
    int64_t max_rows;
    int n_chunks;
    size_t planes, rowscale;   // E4M3 weights + bf16 activations only (else 0 bytes)
    size_t tok_cnt;            // fused combine: arrival counters [T, ceil(H/128)], zeroed with ctrl
    int acc_cols;         // accumulator columns of the widest GEMM tile
};

// Which GEMM kernel a call uses.
struct GemmPlan {
    bool swap;            // weights in the MMA M slot, tokens in N
    int bn;               // Swap-AB: token rows per tile (16..256); normal: 256
};

GemmPlan plan_gemm(const moe_shape_t &s);
// Kernel launches issued by the last entry-point call on this host thread
// (what moe_last_launch_count reports); every entry point resets it.
int &launch_counter();
bool ws_layout(const moe_shape_t &s, WsLayout &L);
int validate_shape(const moe_shape_t *s, bool need_gemm);

// ---- launchers (return cudaError_t of the launch) ----
// the first kernel of a layer call also clears n_zero words at `zero`
cudaError_t launch_route(const moe_shape_t &s, const float *logits, int32_t *ids, float *w,
                         cudaStream_t st, int32_t *zero = nullptr, int n_zero = 0, bool chained = false);
// router logits x . Wg^T and top-k in one launch; tickets [T] must be zero
cudaError_t launch_router(const moe_shape_t &s, const void *x, const void *wg, float *logits,
                          int32_t *tickets, int32_t *ids, float *w, cudaStream_t st, bool chained);
// `chained`: launched by moe_fused_forward after its first kernel (PDL
// launch; the control words and GEMM tile counters were zeroed at the start
// of the call)
// `ticket_zero`: the caller has already cleared ctrl->ticket on this stream
// (skips the memset the two-kernel path otherwise issues)
cudaError_t launch_align(const moe_shape_t &s, const int32_t *ids, int32_t *counts,
                         int32_t *offsets, int32_t *sorted_rows, int32_t *inv, int32_t *chunk_hist,
                         int32_t *chunk_base, Ctrl *ctrl, cudaStream_t st, int *launches,
                         bool chained = false, bool ticket_zero = false);
// Routing + alignment of a batch with T*k <= 1024 routed rows in one block,
// clearing the n_zero words at `zero` (status, ticket, tile and combine
// counters) first.
cudaError_t launch_route_align(const moe_shape_t &s, const float *logits, float *w, int32_t *counts,
                               int32_t *offsets, int32_t *sorted_rows, int32_t *inv, Ctrl *ctrl, int32_t *zero,
                               int n_zero, cudaStream_t st, bool chained);
cudaError_t launch_gather(const moe_shape_t &s, const void *x, const int32_t *sorted_rows,
                          const int32_t *offsets, float a1, void *xp, int64_t max_rows,
                          cudaStream_t st, bool chained = false, bool skip_pad = false);
cudaError_t launch_combine(const moe_shape_t &s, const float *y, const float *w,
                           const int32_t *inv, const int32_t *offsets, void *out,
                           cudaStream_t st, bool chained = false);

// Split bf16 rows [offsets[E+n_shared], K] of `src` into E4M3 planes hi
// (rows 0..) and lo (rows max_rows..) of `planes` with v = scale[row] *
// (hi + lo); see small_kernels.cu.
// Gather + hi/lo split in one pass: the planes of each non-pad slot's token
// row of x [T, H] (lo plane at row max_rows) and its scale.
cudaError_t launch_gather_split(const moe_shape_t &s, const void *x, const int32_t *sorted_rows,
                                const int32_t *offsets, void *planes, float *scale, int64_t max_rows,
                                cudaStream_t st, bool chained);
// sorted_rows (may be NULL): skip the rows of pad slots
cudaError_t launch_split_hilo(const moe_shape_t &s, const void *src, int K, const int32_t *offsets,
                              void *planes, float *scale, int64_t max_rows, cudaStream_t st,
                              bool chained, const int32_t *sorted_rows = nullptr);

struct GemmArgs {
    int mode;                 // 0: gate/up + SwiGLU, 1: down projection
    const void *act;          // xp or h
    const void *wgt;          // w13 or w2
    const float *wscale;
    float ascale, qscale;
    const int32_t *offsets;
    void *out;
    int32_t *status;
    int32_t *counters;
    float *partials;
    int64_t max_rows;
    bool chained;             // PDL launch; counters already zero
    const int32_t *skip_pad_rows = nullptr;   // the layer's sorted_rows: pad slots' rows need no split
    bool planes_ready = false;                // hi/lo path, mode 0: the planes of act were made already
    // Swap-AB mode 0 in the layer: prefetch into L2 this many bytes per CTA of
    // the down projection's weights (next_wgt) once GEMM1's loads are issued
    const void *next_wgt = nullptr;
    long long next_prefetch_bytes = 0;
    bool next_reverse = false;               // GEMM2 walks its tile list backwards (fused combine)
    void *planes;             // E4M3 weights + bf16 activations: hi/lo activation planes
    float *rowscale;          //   [2 * max_rows, K] E4M3 and the scale of each row
    // fused combine (mode 1): slot -> row code; stage rows in ystage [T, k + n_shared, H],
    // count them in tok_cnt [T, n_ct] (zero on entry), write out [T, H] bf16
    bool combine = false;
    const int32_t *sorted_rows = nullptr;
    float *ystage = nullptr;
    int32_t *tok_cnt = nullptr;
    const float *wts = nullptr;
    void *comb_out = nullptr;
    // normal order: which rows of each segment this launch takes (GemmParams)
    int rsplit = 0;
    bool wait_at_end = false;
    int test_stall = 0;       // abort-path test only (GemmParams::test_stall)
};
cudaError_t launch_grouped_gemm(const moe_shape_t &s, const GemmPlan &p, const GemmArgs &a,
                                cudaStream_t st, int *launches, int *host_err);

}  // namespace moe
