// Diagnostic: a bounded wait that nothing satisfies.
//
// Every wait in the library's kernels (on an mbarrier, a copy or another
// role of the same CTA) is bounded by a globaltimer deadline; on expiry the
// kernel records SA_ERR_TIMEOUT in the workspace status word and returns, so
// the context stays usable.  This kernel exercises that path on purpose: one
// thread waits, with the same bounded-wait helper the kernels use, on an
// mbarrier no thread or copy ever arrives on.
#include "sa_internal.h"
#include "tc_ptx.cuh"

namespace sa {
namespace {

__global__ void k_wait_diag(DevStatus *st, unsigned long long timeout_ns)
{
    __shared__ __align__(8) uint64_t bar;
    __shared__ int no_abort;
    if (threadIdx.x == 0) {
        tc::mbar_init(&bar, 1);
        no_abort = 0;
        tc::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint64_t deadline = tc::globaltimer() + timeout_ns;
        if (!tc::mbar_wait(&bar, 0, deadline, &no_abort)) record(st, SA_ERR_TIMEOUT, CHK_WAIT, -1);
    }
}

}  // namespace

cudaError_t launch_wait_diag(DevStatus *st, unsigned long long timeout_ns, cudaStream_t s)
{
    k_wait_diag<<<1, 32, 0, s>>>(st, timeout_ns);
    return cudaGetLastError();
}

}  // namespace sa
