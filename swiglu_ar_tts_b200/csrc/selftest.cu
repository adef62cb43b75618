// Self-test of the bounded mbarrier wait that the streaming kernels use.
//
// One thread arms an mbarrier for 16 transaction bytes that no copy will ever
// deliver, then waits on it with a short limit.  The wait must give up, set
// kDeviceErrTimeout in the library's error word and return, leaving the
// context usable; nothing is in flight, so nothing is left to drain.
#include "common.cuh"
#include "tma.cuh"

namespace arops {
namespace {

__global__ void wait_timeout_kernel(uint64_t timeout_ns, unsigned* err_word, int* waited_out)
{
    __shared__ uint64_t bar;
    const uint32_t b = smem_addr(&bar);
    mbar_init(b, 1);
    mbar_init_fence();
    mbar_arrive_expect_tx(b, 16);  // 16 bytes that never arrive
    const bool ok = mbar_wait(b, 0, timeout_ns);
    if (!ok)
        record_device_error(err_word, kDeviceErrTimeout);
    *waited_out = ok ? 0 : 1;
}

}  // namespace

cudaError_t launch_wait_timeout_selftest(uint64_t timeout_ns, int* waited_out,
                                         cudaStream_t stream)
{
    unsigned* word = nullptr;
    cudaError_t err = device_error_word(&word);
    if (err != cudaSuccess)
        return err;
    return launch(wait_timeout_kernel, dim3(1), dim3(1), 0, stream, timeout_ns, word, waited_out);
}

}  // namespace arops
