// noalloc.cu - moe_align_permute_noalloc: the align/permute step for callers
// that cannot give the library a workspace.
//
// Who needs it: programs whose device memory is owned by an allocator they do
// not control (an inference engine that reserves the GPU's memory at start-up
// and forbids any further cudaMalloc), and latency-critical loops that may not
// call cudaMalloc at all because it can synchronise the device.  Such callers
// can still pass their inputs and outputs, but not an extra scratch buffer.
//
// How: the step's scratch (per-block expert histograms, per-block first slots
// and the control words) lives in one file-scope __device__ array of fixed
// size inside the library.  Every GPU that loads the library holds this array
// until the process exits.  The array's name is only a host-side stand-in, so
// its device address is looked up with cudaGetSymbolAddress once per device,
// on the first call made while that device is current.  The kernels are the
// ones moe_align_permute launches; only where their scratch lives differs.
#include <mutex>

#include "common.cuh"

namespace moe {

constexpr int kNoAllocMaxRows = 64 * kAlignChunk;            // T*k <= 65536 routed rows
constexpr int kNoAllocMaxChunks = kNoAllocMaxRows / kAlignChunk;
constexpr size_t kNoAllocHistBytes = static_cast<size_t>(kNoAllocMaxChunks) * kMaxExpertsTotal * 4;
constexpr size_t kNoAllocCtrlBytes = 256;
constexpr size_t kNoAllocScratchBytes = kNoAllocCtrlBytes + 2 * kNoAllocHistBytes;   // 262,912 bytes
static_assert(sizeof(Ctrl) <= kNoAllocCtrlBytes, "control words must fit");

static __device__ __align__(256) unsigned char g_align_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
static std::mutex g_setup_mutex;
static void *g_scratch_addr[kMaxDevices];

// Device address of g_align_scratch on the current device (looked up once per
// device and kept for the life of the process: a cudaDeviceReset, which
// unloads the library's module, makes the kept address stale).
static int scratch_address(void **addr)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return MOE_ERR_CUDA;
    if (dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_align_scratch) != cudaSuccess || !p) return MOE_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *addr = g_scratch_addr[dev];
    return MOE_OK;
}

}  // namespace moe

using namespace moe;

extern "C" int moe_align_permute_noalloc(const moe_shape_t *shape, const int32_t *ids,
                                         int32_t *counts, int32_t *offsets, int32_t *sorted_rows,
                                         int32_t *inv, int32_t *status, moe_stream_t stream)
{
    int &launches = launch_counter();
    launches = 0;
    int st = validate_shape(shape, false);
    if (st != MOE_OK) return st;
    if (!ids || !counts || !offsets || !sorted_rows || !inv) return MOE_ERR_INVALID_ARG;
    const int64_t R = static_cast<int64_t>(shape->T) * shape->k;
    if (R > kNoAllocMaxRows || shape->E + shape->n_shared > kMaxExpertsTotal) return MOE_ERR_UNSUPPORTED;
    void *base = nullptr;
    st = scratch_address(&base);
    if (st != MOE_OK) return st;
    cudaStream_t sm = reinterpret_cast<cudaStream_t>(stream);
    char *b = static_cast<char *>(base);
    Ctrl *ctrl = reinterpret_cast<Ctrl *>(b);
    int32_t *hist = reinterpret_cast<int32_t *>(b + kNoAllocCtrlBytes);
    int32_t *first = reinterpret_cast<int32_t *>(b + kNoAllocCtrlBytes + kNoAllocHistBytes);
    // the array keeps the previous call's contents: the status word and the
    // blocks-finished ticket (adjacent) must start from zero
    static_assert(offsetof(Ctrl, ticket) == sizeof(int32_t), "status and ticket adjacent");
    if (cudaMemsetAsync(ctrl, 0, 2 * sizeof(int32_t), sm) != cudaSuccess) return MOE_ERR_CUDA;
    if (launch_align(*shape, ids, counts, offsets, sorted_rows, inv, hist, first, ctrl, sm, &launches, false,
                     true) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (status && cudaMemcpyAsync(status, &ctrl->status, sizeof(int32_t), cudaMemcpyDeviceToDevice, sm) !=
                      cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}
