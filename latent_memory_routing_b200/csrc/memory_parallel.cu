// Memory Parallel: merge of the per-shard top-k candidate lists.
//
// Method: "EverMind-AI/MSA: routing top-k compressed documents inside
// attention ..." (hysenlabs.com), §"The 100M-token setup depends on host
// memory as well as two GPUs": the routing keys are split across GPUs, every
// GPU scores the query against its own part, and the partial results are
// reduced into one global selection.  Here a shard is a contiguous range of
// documents; each GPU's local top-k, (score, local document id) in rank
// order, is all-gathered, and this kernel picks the global top-k with the
// same rule as msa_topk_docs (score descending, lower global document index
// first, NaN last, -0 == +0).
//
// Design: one CTA per query.  The world * k candidates become 64-bit keys
// (order-preserving score key << 32 | ~global id): all differ (a document
// lives in one shard), and a larger key is a better rank, so a candidate's
// rank is the number of larger keys -- counted from shared memory.
#include "msa_common.cuh"

namespace msa {
namespace {

constexpr int kMergeThreads = 256;
constexpr int kMaxCands = 4096;

__global__ void __launch_bounds__(kMergeThreads)
merge_shards_kernel(int B, int world, int k, const float* __restrict__ cand_scores,
                    const int32_t* __restrict__ cand_idx, const int32_t* __restrict__ doc_base,
                    int32_t* __restrict__ idx, float* __restrict__ top_scores, int* status) {
  __shared__ unsigned long long keys[kMaxCands];
  const int b = blockIdx.x;
  const int n = world * k;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int r = i / k, j = i % k;
    const int64_t src = ((int64_t)r * B + b) * k + j;
    const float s = cand_scores[src];
    const int64_t id = (int64_t)cand_idx[src] + doc_base[r];
    if (id < 0 || id > 0x7fffffff) record_error(status, MSA_ERR_INVALID_ARG);
    const uint32_t sk = isnan(s) ? 0u : f2o(s + 0.0f);
    keys[i] = ((unsigned long long)sk << 32) | (0xffffffffu - (uint32_t)id);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const unsigned long long ki = keys[i];
    int rank = 0;
    for (int j = 0; j < n; ++j) rank += keys[j] > ki;
    if (rank < k) {
      idx[(int64_t)b * k + rank] = (int32_t)(0xffffffffu - (uint32_t)ki);
      if (top_scores) top_scores[(int64_t)b * k + rank] = cand_scores[((int64_t)(i / k) * B + b) * k + i % k];
    }
  }
}

}  // namespace
}  // namespace msa

extern "C" int msa_topk_merge_shards(int B, int world, int k, const float* cand_scores,
                                     const int32_t* cand_idx, const int32_t* doc_base,
                                     int32_t* idx, float* top_scores, msa_stream_t stream) {
  using namespace msa;
  if (B <= 0 || world <= 0 || k <= 0 || !cand_scores || !cand_idx || !doc_base || !idx)
    return MSA_ERR_INVALID_ARG;
  if ((int64_t)world * k > kMaxCands || B > 0x7fffffff) return MSA_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  merge_shards_kernel<<<(unsigned)B, kMergeThreads, 0, s>>>(
      B, world, k, cand_scores, cand_idx, doc_base, idx, top_scores, device_status_ptr());
  return debug_finish(check_launch(), s);
}
