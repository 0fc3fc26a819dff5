// Input checks of the debug build (compiled only with -DMSA_DEBUG).
//
// The release kernels already reject the data-dependent indexes they meet
// (a document id outside [0, n_docs) in the gather and the fused attention,
// an empty document in chunking, a bad candidate id in the shard merge) by
// recording MSA_ERR_INVALID_ARG in the device status word.  What they trust
// is the shape of the index arrays the caller builds: CSR offsets that never
// decrease and stay inside the tensor they index, and per-query memory
// lengths inside the gathered buffer.  The debug build checks those on the
// device before any kernel reads through them, waits, and returns the error
// from the call that received the bad array.
#include <algorithm>

#include "msa_common.cuh"

#ifdef MSA_DEBUG

namespace msa {
namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads)
check_offsets_kernel(const int64_t* __restrict__ off, int n, int64_t total,
                     int* __restrict__ status) {
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < n; i += stride) {
    const int64_t a = off[i], b = off[i + 1];
    if (a < 0 || b < a || b > total) record_error(status, MSA_ERR_INVALID_ARG);
  }
}

__global__ void __launch_bounds__(kThreads)
check_mem_len_kernel(const int32_t* __restrict__ mem_len, int B, int m_cap,
                     int* __restrict__ status) {
  for (int b = blockIdx.x * kThreads + threadIdx.x; b < B; b += gridDim.x * kThreads) {
    const int32_t m = mem_len[b];
    if (m < 0 || m > m_cap) record_error(status, MSA_ERR_INVALID_ARG);
  }
}

unsigned blocks_for(int64_t n) {
  return (unsigned)std::max<int64_t>(1, std::min<int64_t>((n + kThreads - 1) / kThreads, 1024));
}

// Waits for `s` (unless it is being captured) and returns a CUDA error or
// the status word's error, if any; the word is left as it is.
int wait_and_read(cudaStream_t s) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (int rc = note_cuda(cudaStreamIsCapturing(s, &cs))) return rc;
  if (cs != cudaStreamCaptureStatusNone) return MSA_OK;
  int* st = device_status_ptr();
  if (!st) return note_cuda(cudaErrorInvalidDevice);
  int v = 0;
  if (int rc = note_cuda(cudaMemcpyAsync(&v, st, sizeof(int), cudaMemcpyDeviceToHost, s)))
    return rc;
  if (int rc = note_cuda(cudaStreamSynchronize(s))) return rc;
  return v;
}

}  // namespace

int debug_check_offsets(const int64_t* off, int n, int64_t total, cudaStream_t s) {
  if (!off || n <= 0) return MSA_OK;  // the entry point's own host checks decide
  check_offsets_kernel<<<blocks_for(n), kThreads, 0, s>>>(off, n, total, device_status_ptr());
  if (int rc = check_launch()) return rc;
  return wait_and_read(s);
}

int debug_check_mem_len(const int32_t* mem_len, int B, int m_cap, cudaStream_t s) {
  if (!mem_len || B <= 0) return MSA_OK;
  check_mem_len_kernel<<<blocks_for(B), kThreads, 0, s>>>(mem_len, B, m_cap,
                                                          device_status_ptr());
  if (int rc = check_launch()) return rc;
  return wait_and_read(s);
}

int debug_finish(int rc, cudaStream_t s) {
  if (rc) return rc;
  return wait_and_read(s);
}

}  // namespace msa

#endif  // MSA_DEBUG
