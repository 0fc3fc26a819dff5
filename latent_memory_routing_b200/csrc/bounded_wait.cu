// Failure-detection check of the bounded device waits.
//
// Every pipelined kernel of the library (the routing scan, chunk pooling,
// prefill and decode attention) hands work between its roles through
// mbarriers, and every wait on one is bounded by the global timer: when a
// wait runs out, the kernel records MSA_ERR_TIMEOUT in the device status word
// and its roles wind down without waiting again, so a lost arrival becomes an
// error status the host reads instead of a hung GPU.
//
// bounded_wait_kernel exercises exactly that path on its own: one thread
// initialises an mbarrier that expects one arrival and waits for the
// barrier's first phase with the same bounded wait the pipelines use.  When
// asked not to arrive, nothing completes the phase, the wait expires after
// `limit_ns` and the timeout is recorded; the CTA holds no asynchronous copy
// and no tensor memory, so it simply returns and the context stays usable.
#include "msa_common.cuh"
#include "tc_ptx.cuh"

namespace msa {
namespace {

__global__ void __launch_bounds__(32, 1)
bounded_wait_kernel(uint64_t limit_ns, int arrive, int* __restrict__ status) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  tc::mbar_init(&bar, 1);
  tc::fence_mbar_init();
  if (arrive) tc::mbar_arrive(&bar);
  if (!tc::mbar_wait(&bar, 0, limit_ns)) record_error(status, MSA_ERR_TIMEOUT);
}

}  // namespace
}  // namespace msa

extern "C" int msa_check_bounded_wait(int64_t limit_ns, int arrive, msa_stream_t stream) {
  using namespace msa;
  if (limit_ns < 1000 || limit_ns > 10000000000LL) return MSA_ERR_INVALID_ARG;
  int* status = device_status_ptr();
  if (!status) return note_cuda(cudaErrorInvalidDevice);
  bounded_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      (uint64_t)limit_ns, arrive ? 1 : 0, status);
  return check_launch();
}
