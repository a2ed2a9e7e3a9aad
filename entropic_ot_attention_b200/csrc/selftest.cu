// Self-test of the bounded waits used by every kernel of this library (failure detection).
// A wait that nothing completes must give up once its limit has passed, set the timeout bit
// of the status word, raise the CTA's abort flag and return, so that the kernel ends and the
// context stays usable.  The kernel below exercises the library's own wait routines
// (ptx::mbar_wait on an mbarrier, ptx::grid_wait on a grid-wide counter) with a limit passed
// as a kernel argument; the third case is a control whose wait completes at once.
#include "kernels.cuh"
#include "ptx.cuh"

namespace eot {
namespace {

// scratch words: [0] status word, [1] grid-wide counter (zeroed by the host), [2] result:
// 1 = the wait completed, 2 = the wait gave up.
__global__ void wait_selftest_kernel(int which, unsigned long long limit_ns, uint32_t* scratch) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x != 0) return;
    abort_flag = 0;
    volatile int* ab = &abort_flag;
    uint32_t* status = scratch;
    bool ok;
    if (which == EOT_SELFTEST_GRID) {
        // a grid-wide barrier that waits for one CTA more than the grid holds
        ok = ptx::grid_wait(scratch + 1, gridDim.x + 1, ab, status, limit_ns);
    } else {
        // an mbarrier that expects two arrivals; one arrives (both for the control case)
        const uint32_t b = ptx::smem_u32(&bar);
        ptx::mbar_init(b, 2);
        ptx::mbar_fence_init();
        ptx::mbar_arrive(b);
        if (which == EOT_SELFTEST_CONTROL) ptx::mbar_arrive(b);
        ok = ptx::mbar_wait(b, 0, ab, status, limit_ns);
    }
    scratch[2] = ok ? 1u : 2u;
}

}  // namespace
}  // namespace eot

extern "C" eot_status eot_wait_selftest(int which, uint64_t limit_ns, void* scratch, void* stream) {
    if (which < EOT_SELFTEST_MBARRIER || which > EOT_SELFTEST_CONTROL) return EOT_ERR_INVALID_ARGUMENT;
    if (!scratch || (reinterpret_cast<uintptr_t>(scratch) % 256) != 0) return EOT_ERR_INVALID_ARGUMENT;
    if (limit_ns == 0 || limit_ns > 1000000000ull) return EOT_ERR_INVALID_ARGUMENT;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(scratch, 0, 3 * sizeof(uint32_t), st) != cudaSuccess) return EOT_ERR_CUDA;
    eot::wait_selftest_kernel<<<1, 32, 0, st>>>(which, static_cast<unsigned long long>(limit_ns),
                                                static_cast<uint32_t*>(scratch));
    return cudaGetLastError() == cudaSuccess ? EOT_OK : EOT_ERR_CUDA;
}
