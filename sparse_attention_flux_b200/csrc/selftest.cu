// selftest.cu -- exercises the bounded-wait failure path without faulting or
// hanging the GPU: one thread waits on an mbarrier that nothing ever arrives
// at, using the same bounded wait as every pipeline kernel.  The wait gives up
// after the spin limit, records DEV_ERR_TIMEOUT in the error word and the
// kernel returns, so the host sees FLUX_ERR_TIMEOUT from flux_ctx_check and the
// context stays usable.
#include "common.cuh"
#include "kernels.h"

namespace flux {

namespace {

__global__ void bounded_wait_kernel(DevStatus st, int* waited_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_barrier_init();
  const long long t0 = globaltimer_ns();
  const bool ok = mbar_wait(&bar, 0, st);   // no arrival will ever come
  if (waited_ns) *waited_ns = static_cast<int>((globaltimer_ns() - t0) / 1000);  // microseconds
  if (ok) raise_error(st.err, DEV_ERR_CSR);  // cannot happen: reported as a wrong code
}

}  // namespace

cudaError_t launch_selftest_wait(DevStatus st, int* waited_us, cudaStream_t stream) {
  bounded_wait_kernel<<<1, 32, 0, stream>>>(st, waited_us);
  return cudaGetLastError();
}

}  // namespace flux
