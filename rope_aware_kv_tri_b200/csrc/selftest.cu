// selftest.cu - a device wait that nothing completes, run through the same
// bounded-wait rule as every wait of the library's kernels, so that a test
// can see a wait give up, report TRI_DEVFLAG_TIMEOUT through the caller's
// status word, and leave the CUDA context usable.
//
// No page describes this; it checks the library's own error contract (every
// device wait ends after a time limit and reports instead of hanging).
#include "tri_device.cuh"

namespace tri {

namespace {

// One thread waits either on a shared-memory mbarrier that expects one
// arrival nobody makes (flag == null) or on a global flag only the caller
// could set, for at most kWaitLimitNs (kWaitLimitIters as a backstop).
__global__ void __launch_bounds__(32) selftest_wait_kernel(int32_t* status, const int32_t* flag) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x != 0) return;
    bool done = false;
    if (flag == nullptr) {
        done = mbar_wait_bounded(&bar, 0);
    } else {
        const uint64_t t0 = global_timer_ns();
        for (uint32_t it = 0; it < kWaitLimitIters; ++it) {
            if (ld_acquire_gpu(flag) != 0) {
                done = true;
                break;
            }
            if ((it & 31u) == 0 && global_timer_ns() - t0 > kWaitLimitNs) break;
        }
    }
    if (!done) raise_flag(status, TRI_DEVFLAG_TIMEOUT);
}

}  // namespace

}  // namespace tri

extern "C" tri_status tri_selftest_bounded_wait(int32_t* status, const int32_t* flag, cudaStream_t stream) {
    if (status == nullptr) return TRI_ERR_INVALID;
    if ((reinterpret_cast<uintptr_t>(status) | reinterpret_cast<uintptr_t>(flag)) % alignof(int32_t))
        return TRI_ERR_INVALID;
    tri::selftest_wait_kernel<<<1, 32, 0, stream>>>(status, flag);
    return cudaGetLastError() == cudaSuccess ? TRI_OK : TRI_ERR_CUDA;
}
