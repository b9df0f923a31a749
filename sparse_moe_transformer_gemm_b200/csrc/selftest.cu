// selftest.cu -- moe_selftest_bounded_wait: exercises the library's failure
// detection on the device without faulting, trapping or hanging anything.
//
// Every wait inside the kernels is bounded: a consumer that waits on an
// mbarrier which its producer never completes gives up after a time limit,
// records MOE_ERR_TIMEOUT in the workspace status word and returns, so the
// host reads the error with moe_read_status and the CUDA context stays usable.
// This entry point runs that path on purpose: one thread initialises an
// mbarrier that nothing ever arrives on and waits on it with the same bounded
// wait the kernels use (a caller-chosen limit).
#include "internal.h"
#include "tc.cuh"

namespace {

__global__ void bounded_wait_kernel(unsigned long long limit_ns, int* status) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        abort_flag = 0;
        moe::tc::mbar_init(&bar, 1);
        moe::tc::fence_mbar_init();
        if (!moe::tc::mbar_wait_for(&bar, 0, &abort_flag, limit_ns))
            atomicExch(status, MOE_ERR_TIMEOUT);
    }
}

}  // namespace

extern "C" int moe_selftest_bounded_wait(void* ws, unsigned long long limit_ns, void* stream) {
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MOE_ERR_INVALID_ARG;
    if (limit_ns == 0 || limit_ns > 10000000000ull) return MOE_ERR_INVALID_ARG;  // <= 10 s
    bounded_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
        limit_ns, static_cast<int*>(ws));
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
