// Test-facing probe of the device-side failure detection: every wait in the
// library's kernels (mbarrier waits, grid barriers) gives up after a bounded
// time, records DSPARK_DEV_WAIT_TIMEOUT in the model's status word and lets
// the kernel return, so the context stays usable. dspark_debug_wait_probe
// runs that same bounded mbarrier wait on a barrier that nothing ever
// arrives on, with a short limit, so a test can see the status set and the
// next round run normally.
#include "internal.h"
#include "common.cuh"
#include "tc_ptx.cuh"

namespace dspark {
namespace {

__global__ void wait_probe_kernel(int32_t* status, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    pdl_trigger();
    pdl_wait();
    if (threadIdx.x == 0) {
        abort_flag = 0;
        tc::mbar_init(&bar, 1);          // one arrival expected; none will come
        tc::mbar_fence_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) tc::mbar_wait(&bar, 0u, &abort_flag, status, limit_ns);
    __syncthreads();
}

}  // namespace
}  // namespace dspark

using namespace dspark;

extern "C" int dspark_debug_wait_probe(const dspark_model* m, int32_t limit_us, void* stream) {
    if (!m) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "model is NULL");
    if (limit_us < 1 || limit_us > 2000000) DSPARK_FAIL(DSPARK_ERR_INVALID_ARGUMENT, "limit_us must be in [1, 2000000]");
    cudaError_t e = launch_pdl(wait_probe_kernel, dim3(1), dim3(32), 0, static_cast<cudaStream_t>(stream), m->ws.status,
                               (uint64_t)limit_us * 1000ull);
    if (e != cudaSuccess) DSPARK_FAIL(DSPARK_ERR_CUDA, std::string("wait probe launch: ") + cudaGetErrorString(e));
    return DSPARK_OK;
}
