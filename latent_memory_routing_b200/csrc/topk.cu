// Top-k documents per query, ties to the lower document index.
//
// Method: "EverMind-AI/MSA: routing top-k compressed documents inside
// attention ..." (hysenlabs.com), §"Routing happens inside attention ...":
// the router selects the top-k documents; "深度分析MSA:..." §"五、推理阶段"
// Step 2 (score -> top-k memory).  Equal scores are broken by the lower
// document index, and the output is in rank order.
//
// Design: one 1024-thread CTA per query runs an exact radix select on the
// 32-bit order-preserving key of each score (4 passes of 8 bits, histograms
// in shared memory), which yields the k-th largest key K* and how many of
// the k are strictly above it.  A compaction pass collects the keys > K*,
// an index-ordered pass appends the lowest-index keys == K*, and a bitonic
// sort of the k (score, ~index) 64-bit keys gives rank order.  Scores are
// read from L2 (the whole vector of a 100K-document bank is 400 KB).
#include "msa_common.cuh"

namespace msa {
namespace {

constexpr int kTopkThreads = 1024;
constexpr int kMaxK = 1024;

// NaN ranks below every number; -0.0 and +0.0 are the same score (so their
// tie goes to the lower index, like every other tie).
__device__ __forceinline__ uint32_t score_key(float s) {
  return isnan(s) ? 0u : f2o(s + 0.0f);
}

__global__ void __launch_bounds__(kTopkThreads)
topk_kernel(int n, int k, const float* __restrict__ scores, int32_t* __restrict__ idx_out,
            float* __restrict__ top_out) {
  __shared__ uint32_t hist[256];
  __shared__ unsigned long long cand[kMaxK];
  __shared__ uint32_t s_sel, s_above;
  __shared__ int s_n_gt, s_warp_cnt[32], s_running;
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const float* s = scores + (int64_t)blockIdx.x * n;

  uint32_t prefix = 0, mask = 0;
  int krem = k;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += kTopkThreads) hist[i] = 0;
    __syncthreads();
    // warp-aggregated histogram: scores cluster in few bins, so lanes that
    // share a bin add their count with one shared-memory atomic
    for (int base = 0; base < n; base += kTopkThreads) {
      const int i = base + tid;
      const uint32_t u = i < n ? score_key(__ldg(s + i)) : 0u;
      const bool act = i < n && (u & mask) == prefix;
      const unsigned dig = act ? ((u >> shift) & 255u) : 256u;
      const unsigned peers = __match_any_sync(0xffffffffu, dig);
      if (act && lane == __ffs(peers) - 1) atomicAdd(&hist[dig], (uint32_t)__popc(peers));
    }
    __syncthreads();
    if (warp == 0) {
      // lane l owns digits [8l, 8l+8); suffix sums from the top digit down
      uint32_t own = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) own += hist[8 * lane + j];
      uint32_t suf = own;  // inclusive suffix sum over lanes >= lane
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t o = __shfl_down_sync(0xffffffffu, suf, off);
        if (lane + off < 32) suf += o;
      }
      const uint32_t above_lane = suf - own;  // count in lanes > lane
      const bool here = above_lane < (uint32_t)krem && suf >= (uint32_t)krem;
      if (here) {
        uint32_t cum = above_lane;
        for (int j = 7; j >= 0; --j) {
          const uint32_t hj = hist[8 * lane + j];
          if (cum + hj >= (uint32_t)krem) {
            s_sel = 8 * lane + j;
            s_above = cum;
            break;
          }
          cum += hj;
        }
      }
    }
    __syncthreads();
    prefix |= s_sel << shift;
    mask |= 0xffu << shift;
    krem -= (int)s_above;
    __syncthreads();
  }
  // prefix = key of the k-th best; k - krem keys are strictly greater
  if (tid == 0) { s_n_gt = 0; s_running = 0; }
  __syncthreads();
  for (int i = tid; i < n; i += kTopkThreads) {
    const uint32_t u = score_key(__ldg(s + i));
    if (u > prefix) {
      const int pos = atomicAdd(&s_n_gt, 1);
      cand[pos] = ((unsigned long long)u << 32) | (0xffffffffu - (uint32_t)i);
    }
  }
  __syncthreads();
  const int n_gt = s_n_gt;  // == k - krem
  // lowest-index keys equal to the threshold, in index order
  for (int base = 0; base < n; base += kTopkThreads) {
    if (s_running >= krem) break;  // uniform: read after a barrier
    const int i = base + tid;
    const bool eq = i < n && score_key(__ldg(s + i)) == prefix;
    const unsigned bal = __ballot_sync(0xffffffffu, eq);
    if (lane == 0) s_warp_cnt[warp] = __popc(bal);
    __syncthreads();
    int before = s_running;
    for (int w = 0; w < warp; ++w) before += s_warp_cnt[w];
    const int pos = before + __popc(bal & ((1u << lane) - 1u));
    if (eq && pos < krem)
      cand[n_gt + pos] = ((unsigned long long)prefix << 32) | (0xffffffffu - (uint32_t)i);
    __syncthreads();
    if (tid == 0) {
      int tot = 0;
      for (int w = 0; w < 32; ++w) tot += s_warp_cnt[w];
      s_running += tot;
    }
    __syncthreads();
  }
  // bitonic sort of cand[0..P) descending, P = next power of two >= k
  int P = 1;
  while (P < k) P <<= 1;
  for (int i = k + tid; i < P; i += kTopkThreads) cand[i] = 0ull;
  __syncthreads();
  for (int size = 2; size <= P; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < P; i += kTopkThreads) {
        const int j = i ^ stride;
        if (j > i) {
          const bool desc = (i & size) == 0;
          const unsigned long long a = cand[i], b = cand[j];
          if (desc ? (a < b) : (a > b)) { cand[i] = b; cand[j] = a; }
        }
      }
      __syncthreads();
    }
  }
  for (int r = tid; r < k; r += kTopkThreads) {
    const uint32_t i = 0xffffffffu - (uint32_t)(cand[r] & 0xffffffffull);
    idx_out[(int64_t)blockIdx.x * k + r] = (int32_t)i;
    if (top_out) top_out[(int64_t)blockIdx.x * k + r] = s[i];
  }
}

}  // namespace
}  // namespace msa

extern "C" size_t msa_topk_workspace_size(int B, int n_docs, int k) {
  (void)B; (void)n_docs; (void)k;
  return 0;
}

extern "C" int msa_topk_docs(int B, int n_docs, int k, const float* scores, int32_t* idx,
                             float* top_scores, void* ws, size_t ws_bytes,
                             msa_stream_t stream) {
  (void)ws; (void)ws_bytes;
  if (B <= 0 || n_docs <= 0 || k <= 0 || k > n_docs || k > msa::kMaxK) return MSA_ERR_INVALID_ARG;
  if (!scores || !idx) return MSA_ERR_INVALID_ARG;
  if (B > 65535 * 1024) return MSA_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  msa::topk_kernel<<<B, msa::kTopkThreads, 0, s>>>(n_docs, k, scores, idx, top_scores);
  return msa::check_launch();
}
