// Diagnostic for the forward kernels' failure handling: one CTA runs the same
// bounded mbarrier wait that every pipeline role of fwd_pair.cu uses, on a
// barrier that nothing ever completes.  The wait must run out (~2 s of clock),
// latch the "bounded wait ran out" code in the device error word, raise the
// CTA's abort flag and return, so the kernel exits normally and the context
// stays usable.  No fault, trap or unbounded loop is involved.
#include "fwd_pair_common.cuh"

namespace vsa {
namespace {

__global__ void stall_check_kernel(int* err, int* result)
{
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    // phase 0 of `bar` never completes: no thread arrives on it
    const bool ok = wait_warp(&bar, 0, &abort_flag, err);
    if (threadIdx.x == 0) *result = (ok ? 1 : 0) | (abort_flag != 0 ? 2 : 0);
}

}  // namespace

cudaError_t launch_stall_check(int* err, int* result, cudaStream_t s)
{
    stall_check_kernel<<<1, 32, 0, s>>>(err, result);
    return cudaGetLastError();
}

}  // namespace vsa
