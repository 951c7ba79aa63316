// Diagnostic: the bounded mbarrier wait that every tensor-core kernel of the
// library relies on, run against a barrier that nothing ever arrives on.  The
// wait must give up by itself (after its wall-clock limit) and leave the
// TIMEOUT status for the host, with the GPU context still usable.
#include "twell_device.cuh"

namespace twell {
namespace {

__global__ void k_wait_selftest(int32_t *status, unsigned long long *elapsed_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_word;
  if (threadIdx.x != 0) return;
  abort_word = 0;
  mbar_init(&bar, 1);   // expects one arrival, which never comes
  fence_mbar_init();
  const uint64_t t0 = global_timer_ns();
  const bool ok = mbar_wait(&bar, 0, reinterpret_cast<volatile int *>(&abort_word));
  *elapsed_ns = global_timer_ns() - t0;
  if (!ok) raise_status(status, TWELL_ERR_TIMEOUT);
}

}  // namespace
}  // namespace twell

using namespace twell;

extern "C" twell_status twell_selftest_bounded_wait(int32_t *status, unsigned long long *elapsed_ns,
                                                     void *stream) {
  if (status == nullptr || elapsed_ns == nullptr) return TWELL_ERR_INVALID_ARG;
  k_wait_selftest<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(status, elapsed_ns);
  return cudaGetLastError() == cudaSuccess ? TWELL_OK : TWELL_ERR_CUDA;
}
