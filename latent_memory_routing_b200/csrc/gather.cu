// Context assembly: copy the chunk rows of the selected documents, in rank
// order, into a per-query memory buffer.
//
// Method: "EverMind-AI/MSA: routing top-k compressed documents inside
// attention ..." (hysenlabs.com), §"Memory must be encoded offline before a
// query can reach it" (only the selected K/V are loaded and joined with the
// local context) and §"Routing happens inside attention ..." (their
// compressed K/V are concatenated with the query's local K/V).
//
// Design: kSplit CTAs per (rank, query).  Each finds its destination offset
// from the chunk counts of the higher-ranked documents (k <= 1024 small
// reads), then streams its share of the document's contiguous chunk rows of
// K̄ and V̄ with 16-byte loads and stores -- enough CTAs in flight to cover
// memory latency even for one query.  Rows past m_cap are dropped and the
// overflow is recorded in the device status word.
#include "msa_common.cuh"

namespace msa {
namespace {

constexpr int kSplit = 4;

__global__ void __launch_bounds__(256)
gather_kernel(int k, int n_docs, int row_vecs, const int32_t* __restrict__ idx,
              const int64_t* __restrict__ coff, const uint4* __restrict__ kb,
              const uint4* __restrict__ vb, int m_cap, uint4* __restrict__ km,
              uint4* __restrict__ vm, int32_t* __restrict__ mem_len, int* status) {
  pdl_wait();  // see msa_common.cuh: nothing is touched before the previous grid is done
  pdl_trigger();
  __shared__ int64_t s_off, s_src, s_rows;
  const int r = blockIdx.x / kSplit, part = blockIdx.x % kSplit, b = blockIdx.y;
  const int32_t* ib = idx + (int64_t)b * k;
  if (threadIdx.x < 32) {
    // destination offset = rows of ranks < r (warp-strided sum)
    int64_t off = 0;
    for (int j = threadIdx.x; j < r; j += 32) {
      const int d = ib[j];
      if (d >= 0 && d < n_docs) off += coff[d + 1] - coff[d];
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) off += __shfl_xor_sync(0xffffffffu, off, o);
    if (threadIdx.x == 0) {
      const int d = ib[r];
      int64_t rows = 0, src = 0;
      if (d >= 0 && d < n_docs) {
        src = coff[d];
        rows = coff[d + 1] - src;
      } else {
        record_error(status, MSA_ERR_INVALID_ARG);
      }
      if (r == k - 1 && part == 0) {
        const int64_t total = off + rows;
        mem_len[b] = (int32_t)(total < m_cap ? total : m_cap);
        if (total > m_cap) record_error(status, MSA_ERR_CAPACITY);
      }
      s_off = off;
      s_src = src;
      s_rows = rows;
    }
  }
  __syncthreads();
  int64_t rows = s_rows;
  if (s_off >= m_cap) return;
  if (s_off + rows > m_cap) rows = m_cap - s_off;
  // this CTA's share of the rows
  const int64_t per = (rows + kSplit - 1) / kSplit;
  const int64_t r0 = rows < part * per ? rows : part * per;
  const int64_t r1 = rows < r0 + per ? rows : r0 + per;
  const int64_t n_vec = (r1 - r0) * row_vecs;
  const int64_t off = s_off + r0;
  const uint4* ks = kb + (s_src + r0) * row_vecs;
  const uint4* vs = vb + (s_src + r0) * row_vecs;
  uint4* kd = km + ((int64_t)b * m_cap + off) * row_vecs;
  uint4* vd = vm + ((int64_t)b * m_cap + off) * row_vecs;
  for (int64_t i = threadIdx.x; i < n_vec; i += blockDim.x) {
    const uint4 a = ld_stream16(ks + i);
    const uint4 c = ld_stream16(vs + i);
    kd[i] = a;
    vd[i] = c;
  }
}

}  // namespace
}  // namespace msa

extern "C" int msa_gather_kv(msa_dtype dt, int B, int k, int H, int D, const int32_t* idx,
                             const int64_t* chunk_offsets, int n_docs, const void* k_bar,
                             const void* v_bar, int m_cap, void* k_mem, void* v_mem,
                             int32_t* mem_len, msa_stream_t stream) {
  using namespace msa;
  if (B <= 0 || k <= 0 || n_docs <= 0 || m_cap < 0 || H <= 0 || D <= 0) return MSA_ERR_INVALID_ARG;
  if (k > n_docs || k > 1024) return MSA_ERR_INVALID_ARG;
  if (!idx || !chunk_offsets || !k_bar || !v_bar || !mem_len) return MSA_ERR_INVALID_ARG;
  if (m_cap > 0 && (!k_mem || !v_mem)) return MSA_ERR_INVALID_ARG;
  if (!aligned16(k_bar) || !aligned16(v_bar) || !aligned16(k_mem) || !aligned16(v_mem))
    return MSA_ERR_INVALID_ARG;
  const size_t esz = dt == MSA_F32 ? 4 : (dt == MSA_BF16 ? 2 : 0);
  if (!esz) return MSA_ERR_INVALID_ARG;
  const size_t row_bytes = (size_t)H * D * esz;
  if (row_bytes % 16) return MSA_ERR_UNSUPPORTED;
  if (B > 65535) return MSA_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // the bank's row count is not an argument here: offsets are checked for order only
  if (int rc = debug_check_offsets(chunk_offsets, n_docs, INT64_MAX, s)) return rc;
  const dim3 grid((unsigned)(k * kSplit), (unsigned)B);
  const int rc = launch_pdl(gather_kernel, grid, dim3(256), 0, s, k, n_docs,
                            (int)(row_bytes / 16), idx, chunk_offsets,
                            static_cast<const uint4*>(k_bar), static_cast<const uint4*>(v_bar),
                            m_cap, static_cast<uint4*>(k_mem), static_cast<uint4*>(v_mem), mem_len,
                            device_status_ptr());
  return debug_finish(rc ? rc : check_launch(), s);
}
