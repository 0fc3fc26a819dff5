// Routing: chunk score s[b,c] = max_t (1/H) sum_h cos(Q_r[b,t,h], K̄_r[c,h]),
// document score = max over the document's chunks.
//
// Method: "EverMind-AI/MSA: routing top-k compressed documents inside
// attention ..." (hysenlabs.com), §"Routing happens inside attention, not in
// a retrieval service in front of the model" (cosine similarity, mean over
// heads, then the token-wise maximum); "深度分析MSA:..." §"五、推理阶段"
// Step 2 (Q_r x K̄_r -> score -> top-k).  The pages leave the document-level
// aggregation open; the maximum over the document's chunks is used.
//
// This file holds the query preparation (normalise Q_r per head in fp32 and
// fold in 1/H), the fp32 CUDA-core scan, the final conversion of the
// order-preserving integer maxima to floats, and the C entry point.  The bf16
// scan on the tcgen05 tensor cores lives in route_tc.cu.
#include <algorithm>

#include "msa_common.cuh"
#include "route_tc.cuh"

namespace msa {
namespace {

constexpr float kEps = 1e-12f;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// One warp per (token, head): qhat = q / max(|q|, eps) / H.
// fp32 layout  [NT][H][D]; bf16 (tensor-core) layout [H][n_pad][D], rows
// NT..n_pad-1 zero.  Also sets the ordered-integer score buffers to -inf.
template <typename Tin, typename Tout, bool kHeadMajor>
__global__ void route_prep_kernel(int NT, int H, int D, int n_pad,
                                  const Tin* __restrict__ q_r,
                                  Tout* __restrict__ qhat, uint32_t* doc_u,
                                  int64_t n_doc_u, uint32_t* chunk_u,
                                  int64_t n_chunk_u) {
  pdl_wait();  // see msa_common.cuh: nothing is touched before the previous grid is done
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t n_rows = (int64_t)(kHeadMajor ? n_pad : NT) * H;
  const uint32_t neg_inf = f2o(-INFINITY);
  const int64_t gt = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = gt; i < n_doc_u; i += stride) doc_u[i] = neg_inf;
  if (chunk_u)
    for (int64_t i = gt; i < n_chunk_u; i += stride) chunk_u[i] = neg_inf;
  if (gw >= n_rows) return;
  int n, h;
  if (kHeadMajor) { h = (int)(gw / n_pad); n = (int)(gw % n_pad); }
  else { n = (int)(gw / H); h = (int)(gw % H); }
  float x[4];
  float ss = 0.f;
  const bool live = n < NT;
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const int d = lane + 32 * m;
    x[m] = (live && d < D) ? Elem<Tin>::to_f(q_r[((int64_t)n * H + h) * D + d]) : 0.f;
    ss += x[m] * x[m];
  }
  ss = warp_sum(ss);
  const float sc = 1.0f / (fmaxf(sqrtf(ss), kEps) * (float)H);
  Tout* dst = kHeadMajor ? qhat + ((int64_t)h * n_pad + n) * D
                         : qhat + ((int64_t)n * H + h) * D;
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const int d = lane + 32 * m;
    if (d < D) dst[d] = Elem<Tout>::from_f(x[m] * sc);
  }
}

// fp32 scan on the CUDA cores: one warp per (chunk, query).
template <int D>
__global__ void __launch_bounds__(256)
route_simt_kernel(int T, int H, const float* __restrict__ qhat,
                  const float* __restrict__ kr, int64_t C,
                  const int64_t* __restrict__ coff, int n_docs,
                  uint32_t* doc_u, uint32_t* chunk_u) {
  constexpr int PER = D / 32;
  const int lane = threadIdx.x & 31;
  const int64_t c = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int b = blockIdx.y;
  if (c >= C) return;
  float kv[16][PER];
#pragma unroll
  for (int h = 0; h < 16; ++h) {
    if (h < H) {
      float ss = 0.f;
#pragma unroll
      for (int m = 0; m < PER; ++m) {
        kv[h][m] = kr[(c * H + h) * D + lane + 32 * m];
        ss += kv[h][m] * kv[h][m];
      }
      ss = warp_sum(ss);
      const float inv = 1.0f / fmaxf(sqrtf(ss), kEps);
#pragma unroll
      for (int m = 0; m < PER; ++m) kv[h][m] *= inv;
    }
  }
  float best = -INFINITY;
  for (int t = 0; t < T; ++t) {
    const float* qp = qhat + ((int64_t)b * T + t) * H * D;
    float acc = 0.f;
#pragma unroll
    for (int h = 0; h < 16; ++h) {
      if (h < H) {
#pragma unroll
        for (int m = 0; m < PER; ++m) acc += qp[h * D + lane + 32 * m] * kv[h][m];
      }
    }
    best = fmaxf(best, warp_sum(acc));
  }
  const int64_t d = warp_find_segment(coff, n_docs, c);
  if (lane == 0) {
    const uint32_t o = f2o(best);
    if (chunk_u) atomicMax(chunk_u + (int64_t)b * C + c, o);
    atomicMax(doc_u + (int64_t)b * n_docs + d, o);
  }
}

__global__ void route_finalize_kernel(uint32_t* doc_u, int64_t n_doc_u,
                                      uint32_t* chunk_u, int64_t n_chunk_u) {
  pdl_wait();
  pdl_trigger();
  const int64_t gt = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = gt; i < n_doc_u; i += stride) {
    const float f = o2f(doc_u[i]);
    doc_u[i] = __float_as_uint(f);
  }
  if (chunk_u)
    for (int64_t i = gt; i < n_chunk_u; i += stride) {
      const float f = o2f(chunk_u[i]);
      chunk_u[i] = __float_as_uint(f);
    }
}

size_t qhat_bytes(msa_dtype dt, int B, int T, int H, int D) {
  const int64_t NT = (int64_t)B * T;
  if (dt == MSA_F32) return round_up((size_t)NT * H * D * sizeof(float), 256);
  const int64_t n_pad = route_tc_columns(NT);
  return round_up((size_t)n_pad * H * D * sizeof(__nv_bfloat16), 256);
}

}  // namespace
}  // namespace msa

extern "C" size_t msa_route_workspace_size(msa_dtype dt, int B, int T, int H,
                                           int D) {
  if (B <= 0 || T <= 0 || H <= 0 || D <= 0) return 0;
  return msa::qhat_bytes(dt, B, T, H, D);
}

namespace msa {
namespace {

int route_scores_impl(msa_dtype dt, int B, int T, int H, int D, const void* q_r,
                      const void* kr, int64_t n_chunks, const int64_t* chunk_offsets, int n_docs,
                      float* doc_scores, float* chunk_scores, void* ws, size_t ws_bytes,
                      bool prepared, cudaStream_t s) {
  if (B <= 0 || T <= 0 || H <= 0 || n_docs <= 0 || n_chunks <= 0) return MSA_ERR_INVALID_ARG;
  if (!q_r || !kr || !chunk_offsets || !doc_scores) return MSA_ERR_INVALID_ARG;
  if (!aligned16(kr) || !aligned16(q_r)) return MSA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return MSA_ERR_UNSUPPORTED;
  if (dt != MSA_F32 && dt != MSA_BF16) return MSA_ERR_INVALID_ARG;
  if (prepared && dt != MSA_BF16) return MSA_ERR_UNSUPPORTED;
  if (H > (dt == MSA_BF16 ? 8 : 16)) return MSA_ERR_UNSUPPORTED;
  if ((int64_t)B * T > (1LL << 24)) return MSA_ERR_UNSUPPORTED;
  const size_t need = qhat_bytes(dt, B, T, H, D);
  if (!ws || ws_bytes < need || !aligned16(ws)) return MSA_ERR_WORKSPACE;
  const int NT = B * T;
  uint32_t* doc_u = reinterpret_cast<uint32_t*>(doc_scores);
  uint32_t* chunk_u = reinterpret_cast<uint32_t*>(chunk_scores);
  const int64_t n_doc_u = (int64_t)B * n_docs;
  const int64_t n_chunk_u = chunk_scores ? (int64_t)B * n_chunks : 0;
  const int sms = num_sms();
  int rc;
  if ((rc = debug_check_offsets(chunk_offsets, n_docs, n_chunks, s))) return rc;
  if (dt == MSA_F32) {
    const int64_t rows = (int64_t)NT * H;
    const unsigned blocks = (unsigned)std::min<int64_t>((rows * 32 + 255) / 256 + 1, 1 << 20);
    route_prep_kernel<float, float, false><<<std::max<unsigned>(blocks, (unsigned)sms), 256, 0, s>>>(
        NT, H, D, NT, static_cast<const float*>(q_r), static_cast<float*>(ws), doc_u,
        n_doc_u, chunk_u, n_chunk_u);
    if ((rc = check_launch())) return rc;
    const dim3 grid((unsigned)((n_chunks + 7) / 8), (unsigned)B);
    if (D == 64)
      route_simt_kernel<64><<<grid, 256, 0, s>>>(T, H, static_cast<const float*>(ws),
                                                 static_cast<const float*>(kr), n_chunks,
                                                 chunk_offsets, n_docs, doc_u, chunk_u);
    else
      route_simt_kernel<128><<<grid, 256, 0, s>>>(T, H, static_cast<const float*>(ws),
                                                  static_cast<const float*>(kr), n_chunks,
                                                  chunk_offsets, n_docs, doc_u, chunk_u);
    if ((rc = check_launch())) return rc;
  } else {
    const int n_pad = (int)route_tc_columns(NT);
    const int64_t rows = (int64_t)n_pad * H;
    const unsigned blocks = (unsigned)std::min<int64_t>((rows * 32 + 255) / 256 + 1, 1 << 20);
    if ((rc = launch_pdl(route_prep_kernel<__nv_bfloat16, __nv_bfloat16, true>,
                         dim3(std::max<unsigned>(blocks, (unsigned)sms)), dim3(256), 0, s, NT, H,
                         D, n_pad, static_cast<const __nv_bfloat16*>(q_r),
                         static_cast<__nv_bfloat16*>(ws), doc_u, n_doc_u, chunk_u, n_chunk_u)))
      return rc;
    if ((rc = check_launch())) return rc;
    rc = route_tc_launch(B, T, H, D, static_cast<const __nv_bfloat16*>(ws), n_pad,
                         static_cast<const __nv_bfloat16*>(kr), n_chunks, chunk_offsets, n_docs,
                         doc_u, chunk_u, device_status_ptr(), prepared, s);
    if (rc) return rc;
  }
  rc = launch_pdl(route_finalize_kernel, dim3((unsigned)sms * 4), dim3(256), 0, s, doc_u, n_doc_u,
                  chunk_u, n_chunk_u);
  return debug_finish(rc ? rc : check_launch(), s);
}

}  // namespace
}  // namespace msa

namespace msa {

int route_prep_bf16_launch(int NT, int H, int D, int n_pad, const __nv_bfloat16* q_r,
                           __nv_bfloat16* qhat, cudaStream_t s) {
  const int64_t rows = (int64_t)n_pad * H;
  const unsigned blocks = (unsigned)std::min<int64_t>((rows * 32 + 255) / 256 + 1, 1 << 20);
  route_prep_kernel<__nv_bfloat16, __nv_bfloat16, true><<<blocks, 256, 0, s>>>(
      NT, H, D, n_pad, q_r, qhat, nullptr, 0, nullptr, 0);
  return check_launch();
}

}  // namespace msa

extern "C" int msa_route_scores(msa_dtype dt, int B, int T, int H, int D, const void* q_r,
                                const void* kr_bar, int64_t n_chunks,
                                const int64_t* chunk_offsets, int n_docs, float* doc_scores,
                                float* chunk_scores, void* ws, size_t ws_bytes,
                                msa_stream_t stream) {
  return msa::route_scores_impl(dt, B, T, H, D, q_r, kr_bar, n_chunks, chunk_offsets, n_docs,
                                doc_scores, chunk_scores, ws, ws_bytes, false,
                                reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int msa_route_scores_prepared(msa_dtype dt, int B, int T, int H, int D,
                                         const void* q_r, const void* kr_hat, int64_t n_chunks,
                                         const int64_t* chunk_offsets, int n_docs,
                                         float* doc_scores, float* chunk_scores, void* ws,
                                         size_t ws_bytes, msa_stream_t stream) {
  return msa::route_scores_impl(dt, B, T, H, D, q_r, kr_hat, n_chunks, chunk_offsets, n_docs,
                                doc_scores, chunk_scores, ws, ws_bytes, true,
                                reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int msa_route_prepare_bank(msa_dtype dt, int64_t n_chunks, int H, int D,
                                      const void* kr_bar, void* kr_hat, msa_stream_t stream) {
  using namespace msa;
  if (n_chunks <= 0 || H <= 0 || !kr_bar || !kr_hat) return MSA_ERR_INVALID_ARG;
  if (!aligned16(kr_bar) || !aligned16(kr_hat)) return MSA_ERR_INVALID_ARG;
  if (dt != MSA_BF16 || (D != 64 && D != 128)) return MSA_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return debug_finish(route_prepare_bank_launch(n_chunks * H, D,
                                                static_cast<const __nv_bfloat16*>(kr_bar),
                                                static_cast<__nv_bfloat16*>(kr_hat), s),
                      s);
}
