// csa_wait_probe: a kernel whose one wait can never end, run with a short limit, so that a
// caller can see the library's bounded waits give up with an error status instead of hanging.
//
// Every kernel of the library that waits (on a TMA copy, a tensor-core MMA, a peer warp)
// waits through tc::mbar_wait_limit on a CTA-local mbarrier.  This kernel initialises such
// a barrier for one arrival that nothing makes, waits on its first phase with the caller's
// limit, and on the timeout sets CSA_DEVERR_TIMEOUT and returns.  No copy or MMA is in
// flight, so the CTA exits cleanly and the context stays usable.
#include "common.cuh"
#include "tc.cuh"

namespace csa {
namespace {

__global__ void wait_probe_kernel(uint64_t limit_ns, unsigned* err) {
  __shared__ alignas(8) uint64_t bar;
  if (threadIdx.x == 0) {
    tc::mbar_init(&bar, 1);
    tc::fence_mbar_init();
  }
  __syncthreads();
  const bool ok = tc::mbar_wait_limit(&bar, 0, limit_ns);   // phase 0 never completes
  if (!ok && threadIdx.x == 0) raise_err(err, CSA_DEVERR_TIMEOUT);
}

}  // namespace

cudaError_t launch_wait_probe(uint64_t limit_ns, cudaStream_t st, unsigned* err) {
  note_launch();
  wait_probe_kernel<<<1, 32, 0, st>>>(limit_ns, err);
  return cudaGetLastError();
}

}  // namespace csa
