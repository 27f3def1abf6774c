// selftest.cu -- ret_selftest_wait_timeout: exercises the bounded mbarrier
// wait of the tensor-core kernels on a barrier that nothing completes.
//
// No counterpart in the paper: it is a diagnostic for the failure path.
// One warp initialises an mbarrier that no copy or product will ever
// complete and waits on it through mbar_wait_bounded, the same routine
// every tensor-core kernel waits through, with a caller-chosen limit.  The
// wait gives up, latches RET_ERR_TIMEOUT in the device status word and the
// kernel returns normally, so the context stays usable: exactly what a
// stalled copy or product inside a real kernel would produce.
#include "common.cuh"
#include "launch.h"
#include "tc_util.cuh"

namespace ret {
namespace {

__global__ void __launch_bounds__(32, 1) wait_timeout_kernel(long long limit, int *status) {
    __shared__ __align__(8) uint64_t barrier_word;
    __shared__ int abort_flag;
    const uint32_t bar = tc::smem_u32(&barrier_word);
    if (threadIdx.x == 0) {
        tc::mbar_init(bar, 1);
        abort_flag = 0;
        tc::fence_mbar_init();
    }
    __syncwarp();
    if (threadIdx.x == 0) tc::mbar_wait_bounded(bar, 0, &abort_flag, status, limit);
    __syncwarp();
}

}  // namespace
}  // namespace ret

extern "C" ret_status ret_selftest_wait_timeout(long long cycles, void *stream) {
    if (cycles < 1000 || cycles > 4000000000LL) return RET_ERR_ARG;
    int dev = -1, major = 0, minor = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
        cudaGetLastError();
        return RET_ERR_UNSUPPORTED;
    }
    if (major != 10 || minor != 0) return RET_ERR_UNSUPPORTED;
    int *status = ret::device_status_word();
    if (!status) return RET_ERR_CUDA;
    ret::wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(cycles, status);
    if (cudaGetLastError() != cudaSuccess) return RET_ERR_CUDA;
    ret::note_launches(1);
    return RET_OK;
}
