// la_debug.cu -- a kernel whose bounded wait runs out on purpose, for the tests of the
// timeout path (la_debug_wait_timeout).  Every wait in the tensor-core kernels gives up
// after a time limit, records which wait it was in a fault word and lets the kernel
// return; this kernel takes that path with a short limit on an mbarrier that nothing
// ever arrives on, with no copy or UMMA in flight, so the host can check the report
// (la_device_check) and that the context stays usable.
#include "la_tc.cuh"
#include "la_tc_common.cuh"

namespace la {
namespace tc {

__device__ unsigned int g_debug_fault = 0;

namespace {

// One thread waits, for at most limit_ns, on a fresh mbarrier whose phase never completes.
__global__ void wait_timeout_kernel(unsigned long long limit_ns, int *waited_out) {
    __shared__ uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    fence_mbar_init();
    const bool done = mbar_wait_slow_for(smem_u32(&bar), 0, nullptr, &g_debug_fault, 0x1u, limit_ns);
    if (waited_out) *waited_out = done ? 0 : 1;
}

}  // namespace

unsigned int read_and_clear_debug_fault() {
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_debug_fault, sizeof v) != cudaSuccess) return 0xFFFFFFFFu;
    if (v) cudaMemcpyToSymbol(g_debug_fault, &zero, sizeof zero);
    return v;
}

la_status debug_wait_timeout(unsigned int limit_us, int *waited_out, cudaStream_t st) {
    return launch("debug_wait_timeout", wait_timeout_kernel, dim3(1), dim3(32), 0, st,
                  (unsigned long long)limit_us * 1000ull, waited_out);
}

}  // namespace tc
}  // namespace la

extern "C" la_status la_debug_wait_timeout(unsigned int limit_us, int *waited_out, void *stream) {
    if (limit_us < 1 || limit_us > 1000000u) {
        la::set_error("limit_us must be in [1, 1000000] (got %u)", limit_us);
        return LA_ERR_INVALID_ARG;
    }
    return la::tc::debug_wait_timeout(limit_us, waited_out, (cudaStream_t)stream);
}
