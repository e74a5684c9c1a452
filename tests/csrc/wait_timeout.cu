// wait_timeout.cu -- test-only library (built by tests/test_gpu_wait_timeout.py,
// never linked into libarkattn): makes the library's bounded mbarrier wait run
// out on purpose, without faulting anything.
//
// One thread arms an mbarrier for 16 transaction bytes (arrive.expect_tx) and
// issues no copy, so the phase can never complete.  It then waits with the
// library's own mbar_wait, either with the limit every library kernel uses or
// with a short one, and, when the wait gives up, ORs ARK_DEV_TIMEOUT into the
// status word exactly as the kernels do.  No asynchronous operation refers to
// the barrier, so the CTA can exit with it still armed.
#include "common.cuh"

namespace {

template <uint64_t LimitNs>
__global__ void wait_timeout_kernel(uint32_t* status, unsigned long long* elapsed_ns, int* returned) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x != 0) return;
    ark::mbar_init(&bar, 1);
    ark::fence_mbar_init();
    ark::mbar_arrive_expect_tx(&bar, 16);           // bytes no copy will deliver
    const uint64_t t0 = ark::globaltimer_ns();
    const bool ok = ark::mbar_wait<LimitNs>(&bar, 0);
    *elapsed_ns = ark::globaltimer_ns() - t0;
    if (!ok) ark::report(status, ARK_DEV_TIMEOUT);
    *returned = 1;
}

}  // namespace

// short_limit != 0: a 1 ms limit; 0: the limit every library kernel uses.
extern "C" __attribute__((visibility("default"))) int ark_test_wait_timeout(uint32_t* d_status, unsigned long long* d_elapsed_ns, int* d_returned,
                                     int short_limit, cudaStream_t stream) {
    if (short_limit)
        wait_timeout_kernel<1000000ull><<<1, 32, 0, stream>>>(d_status, d_elapsed_ns, d_returned);
    else
        wait_timeout_kernel<ark::kWaitLimitNs><<<1, 32, 0, stream>>>(d_status, d_elapsed_ns, d_returned);
    return cudaGetLastError() == cudaSuccess ? 0 : 1;
}

// the limit compiled into the library's kernels, for the test's expectations
extern "C" __attribute__((visibility("default"))) unsigned long long ark_test_wait_limit_ns(void) { return ark::kWaitLimitNs; }
