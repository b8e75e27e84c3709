// selftest.cu -- moe_selftest_bounded_wait: the library's bounded-wait
// mechanism exercised on purpose.  Two threads wait on mbarriers that nothing
// completes, through the same mbar_wait_or_abort every kernel uses: the first
// gives up after the wait limit, records MOE_STATUS_TIMEOUT and raises the
// CTA's abort flag; the second gives up then too (on the flag or its own
// limit).  The kernel then returns normally, so the context stays usable.
#include "device_common.cuh"

namespace moe {

namespace {

__global__ void bounded_wait_probe_kernel(int32_t* status, unsigned long long* elapsed_ns) {
    __shared__ uint64_t bars[2];
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    const uint64_t t0 = global_timer_ns();
    const int slot = threadIdx.x == 0 ? 0 : threadIdx.x == 32 ? 1 : -1;
    if (slot >= 0) {
        const bool ok = mbar_wait_or_abort(&bars[slot], 0u, &abort_flag, status);
        elapsed_ns[slot] = ok ? 0ull : global_timer_ns() - t0;
    }
}

}  // namespace

cudaError_t launch_bounded_wait_probe(int32_t* status, unsigned long long* elapsed_ns, cudaStream_t stream) {
    bounded_wait_probe_kernel<<<1, 64, 0, stream>>>(status, elapsed_ns);
    return cudaGetLastError();
}

}  // namespace moe
