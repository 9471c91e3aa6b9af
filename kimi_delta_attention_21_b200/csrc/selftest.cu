// Self-test of the bounded device waits every tensor-core kernel uses.
//
// A one-CTA kernel waits on an mbarrier that nothing ever arrives on, with a
// short limit.  The wait gives up, the kernel records KDA_ERR_TIMEOUT in the
// caller's status word and in the library's timeout counter, and returns: no
// trap, no fault, and the context stays usable.
#include "kda_internal.cuh"
#include "sm100_ptx.cuh"
#include "tma_host.cuh"

namespace kda {
namespace {

__global__ void wait_timeout_kernel(unsigned long long limit_ns, int *status, unsigned int *timeouts) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        sm100::mbar_init(&bar, 1);
        sm100::fence_barrier_init();
    }
    __syncthreads();
    const bool done = sm100::mbar_wait(&bar, 0, limit_ns);  // phase 0 never completes
    __syncthreads();
    if (!done && threadIdx.x == 0) {
        atomicExch(status, (int)KDA_ERR_TIMEOUT);
        if (timeouts) atomicAdd(timeouts, 1u);
    }
}

}  // namespace
}  // namespace kda

extern "C" kda_status_t kda_selftest_wait_timeout(int32_t *dev_status, uint32_t limit_us, void *stream) {
    using namespace kda;
    if (!dev_status) return fail(KDA_ERR_INVALID_ARG, "dev_status is NULL");
    if ((reinterpret_cast<uintptr_t>(dev_status) & 3u) != 0) return fail(KDA_ERR_INVALID_ARG, "dev_status misaligned");
    if (limit_us == 0 || limit_us > 1000000u) return fail(KDA_ERR_INVALID_ARG, "limit_us must be in [1, 1000000]");
    wait_timeout_kernel<<<1, 32, 0, (cudaStream_t)stream>>>((unsigned long long)limit_us * 1000ull, dev_status,
                                                          device_timeout_counter());
    return check_launch("wait_timeout_kernel");
}
