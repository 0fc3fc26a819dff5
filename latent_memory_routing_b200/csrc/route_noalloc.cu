// msa_route_scores_noalloc: msa_route_scores with its workspace taken from a
// fixed scratch array compiled into the library instead of from the caller.
//
// Some callers cannot call cudaMalloc: an engine whose device memory is all
// owned by its own pool allocator (which it does not hand across a C ABI), or
// a latency-critical loop that must not allocate because cudaMalloc may
// synchronise the device.  They still own and pass every input and output;
// only the scratch (the normalised routing queries) lives here.
//
// The scratch is one array per device, kept by every GPU that loads the
// library until the process exits.  All calls on a device share it, so calls
// that overlap on the GPU (different streams, no ordering between them) race
// on it; order them on one stream or with events.  Each call rewrites every
// byte of the scratch it reads before reading it (padded query rows are
// written as zeros), so no state leaks from one call to the next.
#include <mutex>

#include "msa_common.cuh"

namespace msa {
namespace {

// 512 KiB: the bf16 workspace of one full 256-column pass at 8 heads x 128
// dims (msa_route_workspace_size(MSA_BF16, 1, 256, 8, 128)).
constexpr size_t kNoAllocScratchBytes = 512u * 1024u;

static __device__ __align__(256) unsigned char g_route_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_route_scratch on the current device, looked up once
// per device (with that device current) on its first call.
int scratch_ptr(void** out) {
  int dev = 0;
  int rc = note_cuda(cudaGetDevice(&dev));
  if (rc) return rc;
  if (dev < 0 || dev >= kMaxDevices) return MSA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    rc = note_cuda(cudaGetSymbolAddress(&p, g_route_scratch));
    if (rc) {
      // recorded for msa_last_cuda_error(); cleared from the runtime so that
      // the next call's launch check does not report it again
      cudaGetLastError();
      return rc;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return MSA_OK;
}

}  // namespace
}  // namespace msa

extern "C" size_t msa_route_noalloc_scratch_bytes(void) {
  return msa::kNoAllocScratchBytes;
}

extern "C" int msa_route_scores_noalloc(msa_dtype dt, int B, int T, int H, int D,
                                        const void* q_r, const void* kr_bar, int64_t n_chunks,
                                        const int64_t* chunk_offsets, int n_docs,
                                        float* doc_scores, float* chunk_scores,
                                        msa_stream_t stream) {
  const size_t need = msa_route_workspace_size(dt, B, T, H, D);
  if (need == 0) return MSA_ERR_INVALID_ARG;
  if (need > msa::kNoAllocScratchBytes) return MSA_ERR_WORKSPACE;  // shape too large
  void* scratch = nullptr;
  const int rc = msa::scratch_ptr(&scratch);
  if (rc) return rc;
  return msa_route_scores(dt, B, T, H, D, q_r, kr_bar, n_chunks, chunk_offsets, n_docs,
                          doc_scores, chunk_scores, scratch, msa::kNoAllocScratchBytes, stream);
}
