// selftest.cu -- la_selftest_wait_timeout: exercises the bounded-wait failure path.
//
// One CTA initialises an mbarrier that nothing will ever arrive on and waits for it with
// the same bounded wait (ptx::mbar_wait) that every pipeline kernel uses.  After the
// wait's poll limit it records kErrTimeout in the device failure word and the kernel
// returns normally, so the CUDA context stays usable; la_check_status() then reports
// LA_ERR_TIMEOUT.  No other state is touched.
#include "la_internal.cuh"
#include "ptx.cuh"

namespace la {
namespace {

__global__ void wait_timeout_kernel(unsigned *err, int *result) {
    __shared__ uint64_t bar;
    __shared__ int abort;
    if (threadIdx.x == 0) {
        ptx::mbar_init(&bar, 1);
        abort = 0;
        ptx::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const bool ok = ptx::mbar_wait(&bar, 0, &abort, err);   // nobody arrives
        if (result) *result = ok ? 1 : 0;
    }
}

}  // namespace
}  // namespace la

using namespace la;

extern "C" la_status_t la_selftest_wait_timeout(void *stream) {
    timer_reset();
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    timer_begin(st);
    wait_timeout_kernel<<<1, 32, 0, st>>>(device_error_word(), nullptr);
    timer_end(st);
    note_launches(1);
    return cudaGetLastError() == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}
