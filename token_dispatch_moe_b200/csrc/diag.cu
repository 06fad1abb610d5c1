// moe_wait_probe: the library's bounded mbarrier wait, run against a barrier
// that nothing ever completes, so that tests can check the timeout path (the
// kernel gives up, records MOE_ERR_TIMEOUT and returns; the context stays
// usable) without any fault, trap or hang.
#include "common.cuh"
#include "tc.cuh"

namespace moe {
namespace {

__global__ void wait_probe_kernel(int32_t *status, uint64_t limit_ns, int32_t *outcome) {
    __shared__ __align__(8) uint64_t bar;
    const uint32_t b = smem_u32(&bar);
    if (threadIdx.x == 0) {
        mbar_init(b, 1);  // one arrival would complete phase 0; none comes
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    const bool done = mbar_wait_for(b, 0u, status, limit_ns);
    if (threadIdx.x == 0 && outcome) *outcome = done ? 1 : 2;
}

}  // namespace
}  // namespace moe

extern "C" moe_status moe_wait_probe(uint64_t limit_ns, int32_t *d_status, int32_t *d_outcome,
                                     moe_stream_t stream) {
    using namespace moe;
    if (limit_ns == 0 || limit_ns > 1000000000ull) return MOE_ERR_INVALID_ARG;
    wait_probe_kernel<<<1, 32, 0, as_cuda(stream)>>>(d_status, limit_ns, d_outcome);
    return launch_status();
}
