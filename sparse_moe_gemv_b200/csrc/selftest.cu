// redmoe_selftest_wait_limit: exercises the bounded grid-barrier wait that every
// persistent kernel of the library uses, on purpose and with a short limit.
//
// One cooperative launch of one 32-thread block per SM meets at one grid barrier. The
// block numbered `withhold` never arrives, so every other block waits `limit_ns`, records
// ERRBIT_TIMEOUT in the control block's error word and returns. All blocks then leave
// through grid_exit, which resets the barrier counters. No wait in this kernel is
// unbounded: the only loop is the barrier's, which ends at the time limit (or after 2^26
// polls), so the device stays usable and the host reads the outcome with
// redmoe_check_timeout.
#include "common.cuh"
#include "internal.h"

namespace redmoe {

namespace {

constexpr uint64_t SELFTEST_MAX_LIMIT_NS = 1000000000ull;  // 1 s

__global__ void __launch_bounds__(32) wait_selftest_kernel(Control* ctl, int withhold, uint64_t limit_ns) {
    if (int(blockIdx.x) != withhold) grid_barrier(ctl, gridDim.x, 0, limit_ns);
    grid_exit(ctl, gridDim.x);
}

}  // namespace

}  // namespace redmoe

using namespace redmoe;

extern "C" redmoe_status redmoe_selftest_wait_limit(void* workspace, size_t workspace_bytes, int32_t withhold,
                                                    uint64_t limit_ns, void* stream) {
    if (limit_ns == 0 || limit_ns > SELFTEST_MAX_LIMIT_NS) return REDMOE_ERR_INVALID_ARG;
    if (!workspace) {
        workspace = noalloc_scratch_address();
        if (!workspace) return REDMOE_ERR_CUDA;
    } else if (reinterpret_cast<uintptr_t>(workspace) % 256 || workspace_bytes < 256) {
        return REDMOE_ERR_WORKSPACE;
    }
    DevInfo di;
    if (!get_dev_info(&di)) return REDMOE_ERR_CUDA;
    if (withhold >= di.sm_count) return REDMOE_ERR_INVALID_ARG;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(di.sm_count);
    cfg.blockDim = dim3(32);
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    Control* ctl = static_cast<Control*>(workspace);
    const int wh = withhold < 0 ? -1 : withhold;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, wait_selftest_kernel, ctl, wh, limit_ns);
    return e == cudaSuccess ? REDMOE_OK : REDMOE_ERR_CUDA;
}

// ------------------------------------------------------------------------------------
// redmoe_fill_shared_memory: one block per SM takes all the shared memory a block may
// have and fills it with a 32-bit pattern. The next kernel on the stream gets the same
// physical shared memory, so any read of its own shared memory before its data arrived
// returns the pattern (a NaN pattern makes such a read visible in the results) rather
// than a previous launch's identical data.
namespace redmoe {
namespace {

__global__ void __launch_bounds__(1024) fill_shared_kernel(uint32_t pattern, int bytes) {
    extern __shared__ __align__(16) unsigned char fill_smem[];
    uint4* p = reinterpret_cast<uint4*>(fill_smem);
    const uint4 v = make_uint4(pattern, pattern, pattern, pattern);
    for (int i = threadIdx.x; i < bytes / 16; i += blockDim.x) p[i] = v;
    __syncthreads();
}

}  // namespace
}  // namespace redmoe

extern "C" redmoe_status redmoe_fill_shared_memory(uint32_t pattern, void* stream) {
    DevInfo di;
    if (!get_dev_info(&di)) return REDMOE_ERR_CUDA;
    const int bytes = di.max_smem_optin & ~15;
    if (cudaFuncSetAttribute(fill_shared_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
        return REDMOE_ERR_CUDA;
    fill_shared_kernel<<<di.sm_count, 1024, bytes, static_cast<cudaStream_t>(stream)>>>(pattern, bytes);
    return cudaGetLastError() == cudaSuccess ? REDMOE_OK : REDMOE_ERR_CUDA;
}
