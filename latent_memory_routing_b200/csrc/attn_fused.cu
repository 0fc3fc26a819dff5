// Fused context assembly + attention: attention reads the selected
// documents' pooled K/V straight from the bank, with no gathered copy.
//
// Method: "EverMind-AI/MSA: routing top-k compressed documents inside
// attention ..." (hysenlabs.com), §"Memory must be encoded offline before a
// query can reach it" (only the selected documents' K/V are loaded and
// joined with the local context) and §"Routing happens inside attention
// ..." (their compressed K/V are concatenated with the query's local K/V).
//
// Design.  A document's chunk rows are contiguous in the bank, but a
// 128-row memory tile spans several documents and a TMA box has a fixed
// size.  So each document's rows are taken in groups of 8 rows -- one
// 128B-swizzle atom of a 64-element K block, which a TMA box of 8 rows
// writes correctly at any 8-row-aligned place of a tile -- and a query's
// memory is the concatenation of its documents' groups in rank order.  The
// rows of a document's last group that lie past its end are other bank rows:
// the attention masks their scores and zeroes their V in shared memory, so
// they change nothing whatever they hold; memory order does not change
// attention, so the padding changes nothing but the work.
// assemble_groups_kernel (one CTA per query) writes the group list; the
// attention kernels load memory tiles group by group.
#include <algorithm>

#include "attn_tc.cuh"
#include "msa_common.cuh"

namespace msa {
namespace {

constexpr int kAsmThreads = 128;
constexpr int kMaxK = 1024;

__global__ void __launch_bounds__(kAsmThreads)
assemble_groups_kernel(int k, int n_docs, const int32_t* __restrict__ idx,
                       const int64_t* __restrict__ coff, int max_groups,
                       int2* __restrict__ groups, int32_t* __restrict__ n_groups,
                       int32_t* __restrict__ mem_len, int* status) {
  __shared__ int s_pref[kMaxK + 1];
  __shared__ int s_rows[kMaxK];
  __shared__ int s_src[kMaxK];
  const int b = blockIdx.x;
  for (int r = threadIdx.x; r < k; r += blockDim.x) {
    const int d = idx[(int64_t)b * k + r];
    int rows = 0, src = 0;
    if (d >= 0 && d < n_docs) {
      src = (int)coff[d];
      rows = (int)(coff[d + 1] - coff[d]);
    } else {
      record_error(status, MSA_ERR_INVALID_ARG);
    }
    s_rows[r] = rows;
    s_src[r] = src;
  }
  __syncthreads();
  if (threadIdx.x == 0) {  // k <= 1024: a serial prefix over the ranks
    int acc = 0, kept_rows = 0;
    for (int r = 0; r < k; ++r) {
      s_pref[r] = acc;
      const int ng = (s_rows[r] + 7) / 8;
      // rows of the groups that fit in max_groups
      const int fit = max(0, min(ng, max_groups - acc));
      kept_rows += min(s_rows[r], 8 * fit);
      acc += ng;
    }
    s_pref[k] = acc;
    n_groups[b] = min(acc, max_groups);
    if (mem_len) mem_len[b] = kept_rows;
    if (acc > max_groups) record_error(status, MSA_ERR_CAPACITY);
  }
  __syncthreads();
  int2* gq = groups + (int64_t)b * max_groups;
  for (int r = threadIdx.x; r < k; r += blockDim.x) {
    const int rows = s_rows[r], src = s_src[r], p = s_pref[r];
    for (int i = 0; 8 * i < rows && p + i < max_groups; ++i)
      gq[p + i] = make_int2(src + 8 * i, min(8, rows - 8 * i));
  }
}

int max_groups_for(int k, int m_cap) { return (m_cap + 7) / 8 + k; }

struct FusedPlan {
  int max_groups;
  size_t g_bytes, n_bytes, attn_bytes, total;
};

FusedPlan fused_plan(int B, int T, int T_loc, int Hq, int H, int k, int m_cap) {
  FusedPlan p{};
  p.max_groups = max_groups_for(k, m_cap);
  p.g_bytes = round_up((size_t)B * p.max_groups * sizeof(int2), 256);
  p.n_bytes = round_up((size_t)B * sizeof(int32_t), 256);
  p.attn_bytes = T == 1 ? attn_decode_tc_fused_workspace_size(B, T_loc, Hq, H, p.max_groups)
                        : attn_tc_fused_workspace_size(B, T, T_loc, Hq, H, 128, p.max_groups);
  p.total = p.g_bytes + p.n_bytes + p.attn_bytes;
  return p;
}

bool fused_supported(msa_dtype dt, int B, int T, int T_loc, int Hq, int H, int D, int k,
                     int m_cap) {
  if (dt != MSA_BF16 || D != 128) return false;
  if (T == 1) return attn_decode_tc_supported(T, Hq, H, D);
  return attn_tc_supported(B, T, T_loc, Hq, H, D, 8 * max_groups_for(k, m_cap));
}

}  // namespace
}  // namespace msa

extern "C" size_t msa_sparse_attn_fused_workspace_size(msa_dtype dt, int B, int T, int T_loc,
                                                       int Hq, int H, int D, int k, int m_cap) {
  using namespace msa;
  if (B <= 0 || T <= 0 || T_loc < T || H <= 0 || Hq % H || k <= 0 || m_cap < 0) return 0;
  if (!fused_supported(dt, B, T, T_loc, Hq, H, D, k, m_cap)) return 0;
  return fused_plan(B, T, T_loc, Hq, H, k, m_cap).total;
}

extern "C" int msa_sparse_attn_fused(msa_dtype dt, int B, int T, int T_loc, int Hq, int H, int D,
                                     const void* q, const int32_t* idx, int k,
                                     const int64_t* chunk_offsets, int n_docs, const void* k_bar,
                                     const void* v_bar, int64_t n_chunks, int m_cap,
                                     const void* k_loc, const void* v_loc, int pos0,
                                     float rope_base, float scale, void* out, int32_t* mem_len,
                                     void* ws, size_t ws_bytes, msa_stream_t stream) {
  using namespace msa;
  if (B <= 0 || T <= 0 || T_loc < T || H <= 0 || Hq <= 0 || m_cap < 0 || pos0 < 0)
    return MSA_ERR_INVALID_ARG;
  if (k <= 0 || k > kMaxK || k > n_docs || n_docs <= 0 || n_chunks <= 0)
    return MSA_ERR_INVALID_ARG;
  if (!q || !idx || !chunk_offsets || !k_bar || !v_bar || !k_loc || !v_loc || !out)
    return MSA_ERR_INVALID_ARG;
  if (!(rope_base > 0.f)) return MSA_ERR_INVALID_ARG;
  if (Hq % H) return MSA_ERR_UNSUPPORTED;
  if (!fused_supported(dt, B, T, T_loc, Hq, H, D, k, m_cap)) return MSA_ERR_UNSUPPORTED;
  if (n_chunks > INT32_MAX - 8 || B > 0x7fffffff) return MSA_ERR_UNSUPPORTED;
  const FusedPlan p = fused_plan(B, T, T_loc, Hq, H, k, m_cap);
  if ((int64_t)B * p.max_groups * 8 > INT32_MAX) return MSA_ERR_UNSUPPORTED;
  if (!ws || ws_bytes < p.total || !aligned16(ws)) return MSA_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (int rc = debug_check_offsets(chunk_offsets, n_docs, n_chunks, s)) return rc;
  unsigned char* w = static_cast<unsigned char*>(ws);
  int2* groups = reinterpret_cast<int2*>(w);
  int32_t* n_groups = reinterpret_cast<int32_t*>(w + p.g_bytes);
  void* attn_ws = w + p.g_bytes + p.n_bytes;
  assemble_groups_kernel<<<(unsigned)B, kAsmThreads, 0, s>>>(
      k, n_docs, idx, chunk_offsets, p.max_groups, groups, n_groups, mem_len,
      device_status_ptr());
  int rc = check_launch();
  if (rc) return rc;
  const float sc = scale > 0.f ? scale : 1.0f / sqrtf((float)D);
  const float qscale = sc * 1.4426950408889634f;  // log2(e): softmax in base 2
  const FusedMemory fm{groups, n_groups, p.max_groups, k_bar, v_bar, n_chunks};
  if (T == 1)
    rc = attn_decode_tc_launch_fused(B, T_loc, Hq, H, D, q, fm, k_loc, v_loc, pos0, rope_base,
                                     qscale, out, attn_ws, s);
  else
    rc = attn_tc_launch_fused(B, T, T_loc, Hq, H, D, q, fm, k_loc, v_loc, pos0, rope_base, qscale,
                              out, attn_ws, s);
  return debug_finish(rc, s);
}
