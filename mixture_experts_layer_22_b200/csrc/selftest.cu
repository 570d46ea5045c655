// selftest.cu - a check of the failure path that every pipelined kernel of
// the library relies on: a bounded mbarrier wait that runs out reports
// MOE_ERR_TIMEOUT in the workspace status word and the kernel returns, so
// the context stays usable.
#include "common.cuh"
#include "ptx.cuh"

namespace moe {

// One block, two warps, two barriers that nothing arrives on.  Warp 0 waits
// until mbar_wait's time limit and raises the block's abort flag; warp 1,
// waiting on the other barrier, sees the flag and gives up at once -- the
// same abort protocol the grouped GEMM's roles follow.
__global__ void __launch_bounds__(64) wait_timeout_kernel(int32_t *status, int32_t *gave_up)
{
    __shared__ __align__(8) uint64_t s_bar[2];
    __shared__ volatile int s_abort;
    if (threadIdx.x == 0) {
        s_abort = 0;
        mbar_init(smem_u32(&s_bar[0]), 1);
        mbar_init(smem_u32(&s_bar[1]), 1);
        fence_mbar_init();
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) {
        const bool ok = mbar_wait(smem_u32(&s_bar[warp]), 0, &s_abort);
        if (!ok) atomicAdd(gave_up, 1);
    }
    __syncthreads();
    if (threadIdx.x == 0 && s_abort) set_status(status, MOE_ERR_TIMEOUT);
}

}  // namespace moe

using namespace moe;

extern "C" int moe_selftest_wait_timeout(void *ws, int32_t *gave_up, moe_stream_t stream)
{
    if (!ws || !gave_up) return MOE_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(gave_up, 0, sizeof(int32_t), st) != cudaSuccess) return MOE_ERR_CUDA;
    wait_timeout_kernel<<<1, 64, 0, st>>>(static_cast<int32_t *>(ws), gave_up);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
