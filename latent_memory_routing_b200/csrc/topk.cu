// Top-k documents per query, ties to the lower document index.
//
// Method: "EverMind-AI/MSA: routing top-k compressed documents inside
// attention ..." (hysenlabs.com), §"Routing happens inside attention ...":
// the router selects the top-k documents; "深度分析MSA:..." §"五、推理阶段"
// Step 2 (score -> top-k memory).  Equal scores are broken by the lower
// document index, and the output is in rank order.
//
// Design.  A score becomes a 32-bit order-preserving key (NaN lowest,
// -0 == +0), and a candidate a 64-bit key (key << 32 | ~index), so that
// "larger 64-bit key" is exactly "better rank" and all candidates differ.
//   * select: one 1024-thread CTA per (segment, query).  The segment's keys
//     are loaded once into shared memory; an exact 3-pass radix select
//     (11, 11 and 10 bits, warp-aggregated shared histograms) finds the
//     segment's k-th key; a compaction pass takes the keys above it and an
//     index-ordered pass the lowest-index ties.  With one segment per query
//     the k candidates are placed in rank order by counting (each key's rank
//     = number of larger keys; all keys differ) and written as the result;
//     otherwise they go to the workspace.
//   * merge: one CTA per query ranks the segments' candidates the same way
//     (a bitonic sort above 2048 candidates) and writes the first k.
// Very large score vectors whose segments would not fit in shared memory
// keep their keys in global memory (L2) with the same select.
// Small k (<= 32, the routing's top-16): a warp keeps a sorted list of its
// 32 best keys, one per lane, and folds in 32 new keys at a time -- a
// register bitonic sort of the batch (skipped when no key beats the
// list's last), then the top 32 of the two sorted lists by one elementwise
// maximum against the reversed batch and a 5-step bitonic merge.  A
// 512-thread CTA takes a 1024-key segment (its 16 warps' lists merged the
// same way, as a tree); a second kernel merges the segments' lists per
// query.
#include <algorithm>

#include "msa_common.cuh"

namespace msa {
namespace {

constexpr int kThreads = 1024;
constexpr int kMaxK = 1024;
constexpr int kSegSmem = 16384;      // keys per segment held in shared memory
constexpr int kMaxCand = 8192;       // candidates one merge CTA sorts
constexpr int kRankMax = 2048;       // up to this many, merge by counting ranks

// NaN ranks below every number; -0.0 and +0.0 are the same score (so their
// tie goes to the lower index, like every other tie).
__device__ __forceinline__ uint32_t score_key(float s) {
  return isnan(s) ? 0u : f2o(s + 0.0f);
}

__device__ __forceinline__ unsigned long long cand_key(uint32_t key, uint32_t idx) {
  return ((unsigned long long)key << 32) | (0xffffffffu - idx);
}

// Descending bitonic sort of c[0..P) (P a power of two) by the whole block.
__device__ void bitonic_desc(unsigned long long* c, int P) {
  for (int size = 2; size <= P; size <<= 1)
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < P; i += blockDim.x) {
        const int j = i ^ stride;
        if (j > i) {
          const bool desc = (i & size) == 0;
          const unsigned long long a = c[i], b = c[j];
          if (desc ? (a < b) : (a > b)) { c[i] = b; c[j] = a; }
        }
      }
      __syncthreads();
    }
}

struct SmemKeys {
  const uint32_t* k;
  __device__ __forceinline__ uint32_t operator()(int i) const { return k[i]; }
};
struct GlobalKeys {
  const float* s;
  __device__ __forceinline__ uint32_t operator()(int i) const { return score_key(__ldg(s + i)); }
};

constexpr int kBins = 2048;  // 11-bit digits: passes over bits 31..21, 20..10, 9..0

struct SelectShared {
  uint32_t hist[kBins];
  uint32_t sel, above, warp_tot[32];
  int n_gt, running, warp_cnt[32];
};

// Exact top-kk of keys(0..len) into cand[0..kk) (unordered), ties to the
// lower index; indices are offset by base.  Whole block.
template <class Keys>
__device__ void select_topk(const Keys& keys, int len, int kk, uint32_t base,
                            unsigned long long* cand, SelectShared& sh) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t prefix = 0, mask = 0;
  int krem = kk;
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    const uint32_t dmask = pass == 2 ? 1023u : 2047u;
    const int nb = (int)dmask + 1;
    for (int i = tid; i < nb; i += blockDim.x) sh.hist[i] = 0;
    __syncthreads();
    // warp-aggregated histogram: scores cluster in few bins, so lanes that
    // share a bin add their count with one shared-memory atomic
    for (int i0 = 0; i0 < len; i0 += blockDim.x) {
      const int i = i0 + tid;
      const uint32_t u = i < len ? keys(i) : 0u;
      const bool act = i < len && (u & mask) == prefix;
      const unsigned dig = act ? ((u >> shift) & dmask) : 0xffffffffu;
      const unsigned peers = __match_any_sync(0xffffffffu, dig);
      if (act && lane == __ffs(peers) - 1) atomicAdd(&sh.hist[dig], (uint32_t)__popc(peers));
    }
    __syncthreads();
    {
      // the whole block finds the digit: thread t owns bins [bpt*t, bpt*t+bpt);
      // a block suffix sum (warp shuffles, then the 32 warp totals) gives
      // the count above each thread's bins
      const int bpt = (nb + blockDim.x - 1) / blockDim.x;
      const int b0 = tid * bpt;
      uint32_t own = 0;
      for (int j = 0; j < bpt; ++j)
        if (b0 + j < nb) own += sh.hist[b0 + j];
      uint32_t suf = own;  // inclusive suffix sum over lanes >= lane
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t o = __shfl_down_sync(0xffffffffu, suf, off);
        if (lane + off < 32) suf += o;
      }
      if (lane == 0) sh.warp_tot[warp] = suf;
      __syncthreads();
      uint32_t above_warps = 0;
      for (int w = warp + 1; w < (int)(blockDim.x >> 5); ++w) above_warps += sh.warp_tot[w];
      const uint32_t above_me = above_warps + suf - own;  // count in bins above mine
      if (above_me < (uint32_t)krem && above_me + own >= (uint32_t)krem) {
        uint32_t cum = above_me;
        for (int j = bpt - 1; j >= 0; --j) {
          const uint32_t hj = b0 + j < nb ? sh.hist[b0 + j] : 0u;
          if (cum + hj >= (uint32_t)krem) {
            sh.sel = b0 + j;
            sh.above = cum;
            break;
          }
          cum += hj;
        }
      }
    }
    __syncthreads();
    prefix |= sh.sel << shift;
    mask |= dmask << shift;
    krem -= (int)sh.above;
    __syncthreads();
  }
  // prefix = the kk-th best key; kk - krem keys are strictly greater
  if (tid == 0) { sh.n_gt = 0; sh.running = 0; }
  __syncthreads();
  for (int i = tid; i < len; i += blockDim.x) {
    const uint32_t u = keys(i);
    if (u > prefix) cand[atomicAdd(&sh.n_gt, 1)] = cand_key(u, base + (uint32_t)i);
  }
  __syncthreads();
  const int n_gt = sh.n_gt;
  // lowest-index keys equal to the threshold, in index order
  for (int i0 = 0; i0 < len; i0 += blockDim.x) {
    if (sh.running >= krem) break;  // uniform: read after a barrier
    const int i = i0 + tid;
    const bool eq = i < len && keys(i) == prefix;
    const unsigned bal = __ballot_sync(0xffffffffu, eq);
    if (lane == 0) sh.warp_cnt[warp] = __popc(bal);
    __syncthreads();
    int before = sh.running;
    for (int w = 0; w < warp; ++w) before += sh.warp_cnt[w];
    const int pos = before + __popc(bal & ((1u << lane) - 1u));
    if (eq && pos < krem) cand[n_gt + pos] = cand_key(prefix, base + (uint32_t)i);
    __syncthreads();
    if (tid == 0) {
      int tot = 0;
      for (int w = 0; w < (int)(blockDim.x >> 5); ++w) tot += sh.warp_cnt[w];
      sh.running += tot;
    }
    __syncthreads();
  }
}

// Places the n distinct keys c[0..n) in descending order into o[0..min(n,k))
// by counting, for each key, how many keys are larger (its rank): one
// barrier instead of a sorting network.  n <= a few thousand.
__device__ void rank_place(const unsigned long long* c, int n, int k, unsigned long long* o) {
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const unsigned long long x = c[i];
    int rank = 0;
    for (int j = 0; j < n; ++j) rank += c[j] > x;
    if (rank < k) o[rank] = x;
  }
  __syncthreads();
}

__device__ void write_result(const unsigned long long* cand, int k, const float* s,
                             int32_t* idx_out, float* top_out) {
  for (int r = threadIdx.x; r < k; r += blockDim.x) {
    const uint32_t i = 0xffffffffu - (uint32_t)(cand[r] & 0xffffffffull);
    idx_out[r] = (int32_t)i;
    if (top_out) top_out[r] = s[i];
  }
}

// grid (n_seg, B).  cand_ws == nullptr: one segment per query, write result.
template <bool kSmemKeys>
__global__ void __launch_bounds__(kThreads)
topk_select_kernel(int n, int k, int seg_len, const float* __restrict__ scores,
                   int32_t* __restrict__ idx_out, float* __restrict__ top_out,
                   unsigned long long* __restrict__ cand_ws) {
  extern __shared__ __align__(16) unsigned char dyn[];
  __shared__ unsigned long long cand[kMaxK];
  __shared__ unsigned long long ranked[kMaxK];
  __shared__ SelectShared sh;
  const int seg = blockIdx.x, b = blockIdx.y;
  const int s0 = seg * seg_len;
  const int len = min(seg_len, n - s0);
  const int kk = min(k, len);
  const float* s = scores + (int64_t)b * n;
  if (kSmemKeys) {
    uint32_t* keys = reinterpret_cast<uint32_t*>(dyn);
    for (int i = threadIdx.x; i < len; i += blockDim.x) keys[i] = score_key(__ldg(s + s0 + i));
    __syncthreads();
    select_topk(SmemKeys{keys}, len, kk, (uint32_t)s0, cand, sh);
  } else {
    select_topk(GlobalKeys{s + s0}, len, kk, (uint32_t)s0, cand, sh);
  }
  __syncthreads();
  if (cand_ws == nullptr) {
    rank_place(cand, kk, k, ranked);
    write_result(ranked, k, s, idx_out + (int64_t)b * k,
                 top_out ? top_out + (int64_t)b * k : nullptr);
  } else {
    unsigned long long* dst = cand_ws + ((int64_t)b * gridDim.x + seg) * k;
    for (int r = threadIdx.x; r < k; r += blockDim.x) dst[r] = r < kk ? cand[r] : 0ull;
  }
}

// grid (B): the n_seg * k candidates of one query -> its top-k in rank order.
__global__ void __launch_bounds__(kThreads)
topk_merge_kernel(int n, int k, int n_cand, const unsigned long long* __restrict__ cand_ws,
                  const float* __restrict__ scores, int32_t* __restrict__ idx_out,
                  float* __restrict__ top_out) {
  extern __shared__ __align__(16) unsigned char dyn[];
  unsigned long long* c = reinterpret_cast<unsigned long long*>(dyn);
  const int b = blockIdx.x;
  const unsigned long long* src = cand_ws + (int64_t)b * n_cand;
  if (n_cand <= kRankMax) {
    // the segments' pads (key 0) rank last and never reach the first k
    unsigned long long* ranked = c + n_cand;
    for (int i = threadIdx.x; i < n_cand; i += blockDim.x) c[i] = src[i];
    __syncthreads();
    rank_place(c, n_cand, k, ranked);
    write_result(ranked, k, scores + (int64_t)b * n, idx_out + (int64_t)b * k,
                 top_out ? top_out + (int64_t)b * k : nullptr);
    return;
  }
  int P = 1;
  while (P < n_cand) P <<= 1;
  for (int i = threadIdx.x; i < P; i += blockDim.x) c[i] = i < n_cand ? src[i] : 0ull;
  __syncthreads();
  bitonic_desc(c, P);
  write_result(c, k, scores + (int64_t)b * n, idx_out + (int64_t)b * k,
               top_out ? top_out + (int64_t)b * k : nullptr);
}

// ---------------------------------------------------------------- small k
constexpr int kSmallK = 32;
constexpr int kSmallThreads = 512;
constexpr int kSmallWarps = kSmallThreads / 32;
constexpr int kSmallBatches = 2;                           // 32-key batches per warp
constexpr int kSmallSeg = kSmallThreads * kSmallBatches;   // keys per select CTA
constexpr int kMergeSmemLists = 160;                       // lists a merge CTA stages (40 KB)

__device__ __forceinline__ unsigned long long umax64(unsigned long long a, unsigned long long b) {
  return a > b ? a : b;
}
__device__ __forceinline__ unsigned long long umin64(unsigned long long a, unsigned long long b) {
  return a < b ? a : b;
}

// Sorts one key per lane, descending across lanes 0..31 (bitonic network).
__device__ __forceinline__ unsigned long long warp_sort_desc(unsigned long long x, int lane) {
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1)
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      const unsigned long long y = __shfl_xor_sync(0xffffffffu, x, j);
      const bool desc = (lane & k) == 0 || k == 32;  // this block's direction
      const bool lower = (lane & j) == 0;
      x = (lower == desc) ? umax64(x, y) : umin64(x, y);
    }
  return x;
}

// Top 32 of two descending lists (one key per lane each), descending.
__device__ __forceinline__ unsigned long long warp_merge_desc(unsigned long long a,
                                                              unsigned long long b, int lane) {
  // a descending, b reversed ascending: their elementwise maximum is the top
  // 32 of the union, as a bitonic sequence
  unsigned long long z = umax64(a, __shfl_sync(0xffffffffu, b, 31 - lane));
#pragma unroll
  for (int j = 16; j > 0; j >>= 1) {
    const unsigned long long y = __shfl_xor_sync(0xffffffffu, z, j);
    z = (lane & j) == 0 ? umax64(z, y) : umin64(z, y);
  }
  return z;
}

// The block's per-warp sorted lists lists[0..kSmallWarps) -> lists[0], by a
// tree of pairwise merges (log2(warps) levels).
__device__ __forceinline__ unsigned long long block_merge_lists(
    unsigned long long (*lists)[32], int warp, int lane) {
#pragma unroll
  for (int half = kSmallWarps / 2; half >= 1; half >>= 1) {
    __syncthreads();
    if (warp < half) lists[warp][lane] = warp_merge_desc(lists[warp][lane],
                                                         lists[warp + half][lane], lane);
  }
  __syncthreads();
  return lists[0][lane];
}

__device__ __forceinline__ void write_small(unsigned long long key, int lane, int k, int64_t row,
                                            const float* __restrict__ s,
                                            int32_t* __restrict__ idx_out,
                                            float* __restrict__ top_out) {
  if (lane < k) {
    const uint32_t i = 0xffffffffu - (uint32_t)(key & 0xffffffffull);
    idx_out[row * k + lane] = (int32_t)i;
    if (top_out) top_out[row * k + lane] = s[i];
  }
}

// grid (n_seg, B).  Each warp folds its 64 keys into a sorted top 32 (a
// batch's sort is skipped when none of it beats the list's last); the
// block merges the 16 lists.  n_seg == 1 writes the result, otherwise the
// segment's sorted list goes to seg_out [B][n_seg][32].
__global__ void __launch_bounds__(kSmallThreads)
topk_small_select_kernel(int n, int k, const float* __restrict__ scores,
                         int32_t* __restrict__ idx_out, float* __restrict__ top_out,
                         unsigned long long* __restrict__ seg_out) {
  pdl_wait();  // see msa_common.cuh: nothing is touched before the previous grid is done
  pdl_trigger();
  __shared__ unsigned long long lists[kSmallWarps][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int b = blockIdx.y;
  const float* s = scores + (int64_t)b * n;
  const int64_t base = (int64_t)blockIdx.x * kSmallSeg + warp * 32 * kSmallBatches;
  unsigned long long key[kSmallBatches];
#pragma unroll
  for (int i = 0; i < kSmallBatches; ++i) {  // all loads in flight first
    const int64_t e = base + i * 32 + lane;
    key[i] = e < n ? cand_key(score_key(__ldg(s + e)), (uint32_t)e) : 0ull;
  }
  unsigned long long list = warp_sort_desc(key[0], lane);
#pragma unroll
  for (int i = 1; i < kSmallBatches; ++i) {
    const unsigned long long thr = __shfl_sync(0xffffffffu, list, 31);
    if (__any_sync(0xffffffffu, key[i] > thr))
      list = warp_merge_desc(list, warp_sort_desc(key[i], lane), lane);
  }
  lists[warp][lane] = list;
  const unsigned long long acc = block_merge_lists(lists, warp, lane);
  if (warp == 0) {
    if (gridDim.x == 1) write_small(acc, lane, k, b, s, idx_out, top_out);
    else seg_out[((int64_t)b * gridDim.x + blockIdx.x) * 32 + lane] = acc;
  }
}

// grid (B): the n_seg sorted lists of one query -> its top-k in rank order.
// Up to kMergeSmemLists lists are staged in shared memory by the whole block
// first (one round of loads), then each warp folds its share and the block
// merges the warps' lists.
__global__ void __launch_bounds__(kSmallThreads)
topk_small_merge_kernel(int n, int k, int n_seg, const unsigned long long* __restrict__ seg_in,
                        const float* __restrict__ scores, int32_t* __restrict__ idx_out,
                        float* __restrict__ top_out) {
  pdl_wait();
  pdl_trigger();
  __shared__ unsigned long long staged[kMergeSmemLists * 32];
  __shared__ unsigned long long lists[kSmallWarps][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int b = blockIdx.x;
  const unsigned long long* src = seg_in + (int64_t)b * n_seg * 32;
  unsigned long long acc = 0ull;
  for (int s0 = 0; s0 < n_seg; s0 += kMergeSmemLists) {
    const int ns = min(kMergeSmemLists, n_seg - s0);
    __syncthreads();  // the previous round's lists have been read
    for (int e = threadIdx.x; e < ns * 32; e += kSmallThreads) staged[e] = src[(int64_t)s0 * 32 + e];
    __syncthreads();
    for (int sg = warp; sg < ns; sg += kSmallWarps) {
      const unsigned long long x = staged[sg * 32 + lane];
      const unsigned long long thr = __shfl_sync(0xffffffffu, acc, 31);
      if (__any_sync(0xffffffffu, x > thr)) acc = warp_merge_desc(acc, x, lane);
    }
  }
  lists[warp][lane] = acc;
  acc = block_merge_lists(lists, warp, lane);
  if (warp == 0) write_small(acc, lane, k, b, scores + (int64_t)b * n, idx_out, top_out);
}

struct TopkPlan {
  int seg_len, n_seg;
  bool smem_keys, small;
  size_t ws_bytes;
};

TopkPlan plan(int B, int n, int k) {
  TopkPlan p{};
  if (k <= kSmallK && (int64_t)(n + kSmallSeg - 1) / kSmallSeg <= 65535) {
    p.small = true;
    p.seg_len = kSmallSeg;
    p.n_seg = (n + kSmallSeg - 1) / kSmallSeg;
    p.ws_bytes = p.n_seg > 1 ? (size_t)B * p.n_seg * kSmallK * sizeof(unsigned long long) : 0;
    return p;
  }
  if (n <= kSegSmem) {
    p.seg_len = n;
    p.n_seg = 1;
    p.smem_keys = true;
    return p;
  }
  // about 4096 keys per segment, fewer segments when k is large
  int seg = 4096;
  const int max_seg_count = std::max(1, kMaxCand / k);
  if ((n + seg - 1) / seg > max_seg_count) seg = (n + max_seg_count - 1) / max_seg_count;
  seg = (seg + 1023) / 1024 * 1024;
  p.seg_len = seg;
  p.n_seg = (n + seg - 1) / seg;
  p.smem_keys = seg <= kSegSmem;
  if (p.n_seg == 1) return p;
  p.ws_bytes = (size_t)B * p.n_seg * k * sizeof(unsigned long long);
  return p;
}

}  // namespace
}  // namespace msa

extern "C" size_t msa_topk_workspace_size(int B, int n_docs, int k) {
  if (B <= 0 || n_docs <= 0 || k <= 0 || k > n_docs || k > msa::kMaxK) return 0;
  return msa::plan(B, n_docs, k).ws_bytes;
}

static int topk_docs_body(int B, int n_docs, int k, const float* scores, int32_t* idx,
                          float* top_scores, void* ws, size_t ws_bytes, msa_stream_t stream) {
  using namespace msa;
  if (B <= 0 || n_docs <= 0 || k <= 0 || k > n_docs || k > kMaxK) return MSA_ERR_INVALID_ARG;
  if (!scores || !idx) return MSA_ERR_INVALID_ARG;
  if (B > 65535) return MSA_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const TopkPlan p = plan(B, n_docs, k);
  if (p.ws_bytes && (!ws || ws_bytes < p.ws_bytes || !aligned16(ws))) return MSA_ERR_WORKSPACE;
  unsigned long long* cand = p.n_seg > 1 ? static_cast<unsigned long long*>(ws) : nullptr;
  const dim3 grid((unsigned)p.n_seg, (unsigned)B);
  int rc;
  if (p.small) {
    rc = launch_pdl(topk_small_select_kernel, grid, dim3(kSmallThreads), 0, s, n_docs, k, scores,
                    idx, top_scores, cand);
    if (rc || (rc = check_launch()) || p.n_seg == 1) return rc;
    rc = launch_pdl(topk_small_merge_kernel, dim3(B), dim3(kSmallThreads), 0, s, n_docs, k,
                    p.n_seg, cand, scores, idx, top_scores);
    return rc ? rc : check_launch();
  }
  if (p.smem_keys) {
    const size_t smem = (size_t)p.seg_len * sizeof(uint32_t);
    rc = ensure_smem_attr(reinterpret_cast<const void*>(topk_select_kernel<true>), (int)smem);
    if (rc) return rc;
    topk_select_kernel<true><<<grid, kThreads, smem, s>>>(n_docs, k, p.seg_len, scores, idx,
                                                           top_scores, cand);
  } else {
    topk_select_kernel<false><<<grid, kThreads, 0, s>>>(n_docs, k, p.seg_len, scores, idx,
                                                         top_scores, cand);
  }
  if ((rc = check_launch())) return rc;
  if (p.n_seg == 1) return MSA_OK;
  const int n_cand = p.n_seg * k;
  int P = 1;
  while (P < n_cand) P <<= 1;
  const size_t smem = (size_t)std::max(P, n_cand <= kRankMax ? n_cand + k : 0) *
                      sizeof(unsigned long long);
  rc = ensure_smem_attr(reinterpret_cast<const void*>(topk_merge_kernel), (int)smem);
  if (rc) return rc;
  topk_merge_kernel<<<B, kThreads, smem, s>>>(n_docs, k, n_cand, cand, scores, idx, top_scores);
  return check_launch();
}

extern "C" int msa_topk_docs(int B, int n_docs, int k, const float* scores, int32_t* idx,
                             float* top_scores, void* ws, size_t ws_bytes,
                             msa_stream_t stream) {
  return msa::debug_finish(
      topk_docs_body(B, n_docs, k, scores, idx, top_scores, ws, ws_bytes, stream),
      reinterpret_cast<cudaStream_t>(stream));
}
