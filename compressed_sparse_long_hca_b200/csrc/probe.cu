// Test helper behind csa_debug_wait_timeout: one thread block waits, through
// the bounded-wait routine every tensor-core kernel of the library uses for
// its mbarriers, on a barrier that nothing ever arrives on.  The wait gives
// up after its limit, the block records a timeout in the device error word
// and returns.  This shows on the device that a bounded wait ends and that
// the context stays usable afterwards; nothing faults, traps or spins
// without a limit.
#include "common.cuh"
#include "tc.cuh"

namespace csa {

__global__ void __launch_bounds__(32) wait_probe_kernel(Layout L, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    tc::mbar_init(&bar, 1);
    tc::fence_mbar_init();
  }
  __syncthreads();
  const bool done = tc::mbar_wait(&bar, 0, limit_ns);   // phase 0 never completes
  if (!done && threadIdx.x == 0) set_err(L, kErrTimeout, 5000000);
}

cudaError_t launch_wait_probe(const Layout& L, uint64_t limit_ns, cudaStream_t st) {
  wait_probe_kernel<<<1, 32, 0, st>>>(L, limit_ns);
  note_launch();
  return cudaGetLastError();
}

}  // namespace csa
