// nosa_diag.cu -- a check of the error path that every bounded device wait takes.
//
// Each pipeline of the library waits on mbarriers with a bound (mbar_wait); a
// wait that runs out sets NOSA_EFLAG_TIMEOUT in the state's error word and the
// kernel drains and returns, so the context stays usable.  This entry point
// runs that same wait on a phase that no thread ever completes, with a short
// bound, so a test can observe the error word without any fault or hang.
#include "nosa_internal.cuh"

namespace nosa {
namespace {
__global__ void wait_timeout_kernel(uint32_t *err, long long limit) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);  // one arrival expected; none comes
    fence_mbar_init();
    if (!mbar_wait(&bar, 0, limit)) set_error(err, NOSA_EFLAG_TIMEOUT);
}
}  // namespace
}  // namespace nosa

extern "C" int nosa_check_wait_timeout(uint32_t *err, int64_t max_cycles, void *stream) {
    if (!err || max_cycles <= 0 || max_cycles > nosa::kWaitCycles) return NOSA_ERR_ARG;
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, err) != cudaSuccess) {
        cudaGetLastError();
        return NOSA_ERR_PTR;
    }
    if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged) return NOSA_ERR_PTR;
    nosa::wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(err, (long long)max_cycles);
    return cudaGetLastError() == cudaSuccess ? NOSA_OK : NOSA_ERR_CUDA;
}
