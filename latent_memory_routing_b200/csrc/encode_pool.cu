// Memory encoding: document-wise RoPE on token K fused with 64-token chunk
// means of K, V and K_r.
//
// Method: "EverMind-AI/MSA: routing top-k compressed documents inside
// attention ..." (hysenlabs.com), §"Document-wise RoPE resets every document
// to position zero" and §"Memory must be encoded offline before a query can
// reach it"; "深度分析MSA:把超长文档组织成可检索内部记忆的工程路径",
// §"三、文档如何变成 memory" / "2. chunk 压缩" (64 tokens per chunk,
// K -> K̄, V -> V̄, K_r -> K̄_r by mean pooling, 180 tokens -> 3 chunks).
//
// Design (HBM-bound stream): one CTA per chunk, looping over the L layers so
// the chunk's RoPE table is built once.  Each thread owns two 16-byte vectors
// of one head -- elements [v*VEC, v*VEC+VEC) and the rotate-half partners at
// +D/2 -- so the rotation needs no data exchange; R token rows are in flight
// per CTA.  Loads are 16-byte, coalesced and L1-bypassing; sums are fp32;
// the R partial sums are combined through shared memory and each output row
// is written once with 16-byte stores.
#include "msa_common.cuh"

namespace msa {
namespace {

constexpr int kEncThreads = 256;
constexpr int kMaxChunk = 64;

template <typename T, int D>
__global__ void __launch_bounds__(kEncThreads)
encode_pool_kernel(int L, int64_t n_tok, int n_docs, int H, int R,
                   const T* __restrict__ k_tok, const T* __restrict__ v_tok,
                   const T* __restrict__ kr_tok,
                   const int64_t* __restrict__ tok_off,
                   const int64_t* __restrict__ chunk_off, int64_t n_chunks,
                   double base, int chunk, T* __restrict__ k_bar,
                   T* __restrict__ v_bar, T* __restrict__ kr_bar) {
  constexpr int VEC = Vec16<T>::N;
  constexpr int HALF = D / 2;
  constexpr int UPH = HALF / VEC;  // pair-vectors per head
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float2* cs_tab = reinterpret_cast<float2*>(smem_raw);           // [64][HALF]
  float* red = reinterpret_cast<float*>(cs_tab + kMaxChunk * HALF);  // [R][3][H*D]
  __shared__ double w_tab[HALF];
  __shared__ int64_t s_tok0, s_p0;
  __shared__ int s_rows;

  const int tid = threadIdx.x;
  const int U = H * UPH;
  const int u = tid % U, r = tid / U;
  const int h = u / UPH, v = u % UPH;
  const int64_t c = blockIdx.x;
  const int64_t row_elems = (int64_t)H * D;

  if (tid < 32) {
    const int64_t d = warp_find_segment(chunk_off, n_docs, c);
    if (tid == 0) {
      const int64_t j = c - chunk_off[d];
      const int64_t t0 = tok_off[d] + j * chunk;
      const int64_t left = tok_off[d + 1] - t0;
      s_tok0 = t0;
      s_p0 = j * chunk;  // position of the chunk's first token in its doc
      s_rows = (int)(left < 0 ? 0 : (left < chunk ? left : chunk));
    }
  }
  for (int i = tid; i < HALF; i += blockDim.x) w_tab[i] = rope_inv_freq(base, i, D);
  __syncthreads();
  const int rows = s_rows;
  const int64_t tok0 = s_tok0, p0 = s_p0;
  for (int e = tid; e < rows * HALF; e += blockDim.x) {
    const int t = e / HALF, i = e - (e / HALF) * HALF;
    cs_tab[e] = rope_cs(p0 + t, w_tab[i]);
  }
  __syncthreads();

  const float inv_n = rows > 0 ? 1.0f / (float)rows : 0.f;
  const int64_t col_lo = (int64_t)h * D + v * VEC;
  for (int l = 0; l < L; ++l) {
    float ak[2][VEC], av[2][VEC], ar[2][VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
      ak[0][e] = ak[1][e] = av[0][e] = av[1][e] = ar[0][e] = ar[1][e] = 0.f;
    }
    if (r < R) {
      const int64_t layer_row0 = (int64_t)l * n_tok + tok0;
#pragma unroll 2
      for (int t = r; t < rows; t += R) {
        const int64_t off = (layer_row0 + t) * row_elems + col_lo;
        const uint4 k0 = ld_stream16(k_tok + off), k1 = ld_stream16(k_tok + off + HALF);
        const uint4 v0 = ld_stream16(v_tok + off), v1 = ld_stream16(v_tok + off + HALF);
        const uint4 r0 = ld_stream16(kr_tok + off), r1 = ld_stream16(kr_tok + off + HALF);
        float x1[VEC], x2[VEC], f[VEC];
        Vec16<T>::unpack(k0, x1);
        Vec16<T>::unpack(k1, x2);
        const float2* cs = cs_tab + t * HALF + v * VEC;
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
          const float2 q = cs[e];
          ak[0][e] += x1[e] * q.x - x2[e] * q.y;
          ak[1][e] += x2[e] * q.x + x1[e] * q.y;
        }
        Vec16<T>::unpack(v0, f);
#pragma unroll
        for (int e = 0; e < VEC; ++e) av[0][e] += f[e];
        Vec16<T>::unpack(v1, f);
#pragma unroll
        for (int e = 0; e < VEC; ++e) av[1][e] += f[e];
        Vec16<T>::unpack(r0, f);
#pragma unroll
        for (int e = 0; e < VEC; ++e) ar[0][e] += f[e];
        Vec16<T>::unpack(r1, f);
#pragma unroll
        for (int e = 0; e < VEC; ++e) ar[1][e] += f[e];
      }
      float* my = red + (int64_t)r * 3 * row_elems;
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        my[col_lo + e] = ak[0][e];
        my[col_lo + HALF + e] = ak[1][e];
        my[row_elems + col_lo + e] = av[0][e];
        my[row_elems + col_lo + HALF + e] = av[1][e];
        my[2 * row_elems + col_lo + e] = ar[0][e];
        my[2 * row_elems + col_lo + HALF + e] = ar[1][e];
      }
    }
    __syncthreads();
    const int64_t out_row = ((int64_t)l * n_chunks + c) * row_elems;
    for (int64_t e0 = (int64_t)tid * VEC; e0 < 3 * row_elems;
         e0 += (int64_t)blockDim.x * VEC) {
      const int tensor = (int)(e0 / row_elems);
      const int64_t col = e0 - tensor * row_elems;
      float o[VEC];
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        float s = 0.f;
        for (int rr = 0; rr < R; ++rr) s += red[(int64_t)rr * 3 * row_elems + e0 + e];
        o[e] = s * inv_n;
      }
      T* dst = tensor == 0 ? k_bar : (tensor == 1 ? v_bar : kr_bar);
      st16(dst + out_row + col, Vec16<T>::pack(o));
    }
    __syncthreads();
  }
}

__global__ void chunk_offsets_kernel(int n_docs, const int64_t* __restrict__ tok_off,
                                     int chunk, int64_t* __restrict__ chunk_off,
                                     int* status) {
  __shared__ int64_t part[1024];
  const int tid = threadIdx.x;
  const int per = (n_docs + blockDim.x - 1) / blockDim.x;
  const int d0 = tid * per;
  const int d1 = min(d0 + per, n_docs);
  int64_t s = 0;
  for (int d = d0; d < d1; ++d) {
    const int64_t len = tok_off[d + 1] - tok_off[d];
    if (len <= 0) record_error(status, MSA_ERR_INVALID_ARG);
    else s += (len + chunk - 1) / chunk;
  }
  part[tid] = s;
  __syncthreads();
  for (int off = 1; off < (int)blockDim.x; off <<= 1) {  // inclusive scan
    const int64_t add = tid >= off ? part[tid - off] : 0;
    __syncthreads();
    part[tid] += add;
    __syncthreads();
  }
  int64_t run = part[tid] - s;  // exclusive
  if (tid == 0) chunk_off[0] = 0;
  for (int d = d0; d < d1; ++d) {
    const int64_t len = tok_off[d + 1] - tok_off[d];
    if (len > 0) run += (len + chunk - 1) / chunk;
    chunk_off[d + 1] = run;
  }
}

template <typename T, int D>
int launch_encode(int L, int64_t n_tok, int n_docs, int H, const void* k,
                  const void* v, const void* kr, const int64_t* toff,
                  const int64_t* coff, int64_t n_chunks, float base, int chunk,
                  void* kb, void* vb, void* rb, cudaStream_t s) {
  constexpr int VEC = Vec16<T>::N;
  const int U = H * (D / 2 / VEC);
  const int R = U >= kEncThreads ? 1 : kEncThreads / U;
  const int threads = U * R;
  if (threads > kEncThreads) return MSA_ERR_UNSUPPORTED;
  const size_t smem = sizeof(float2) * kMaxChunk * (D / 2) +
                      sizeof(float) * (size_t)R * 3 * H * D;
  auto kern = encode_pool_kernel<T, D>;
  int rc = ensure_smem_attr(reinterpret_cast<const void*>(kern), (int)smem);
  if (rc) return rc;
  if (n_chunks == 0) return MSA_OK;
  kern<<<(unsigned)n_chunks, threads, smem, s>>>(
      L, n_tok, n_docs, H, R, static_cast<const T*>(k), static_cast<const T*>(v),
      static_cast<const T*>(kr), toff, coff, n_chunks, (double)base, chunk,
      static_cast<T*>(kb), static_cast<T*>(vb), static_cast<T*>(rb));
  return check_launch();
}

}  // namespace
}  // namespace msa

extern "C" int msa_chunk_offsets(int n_docs, const int64_t* tok_offsets,
                                 int chunk, int64_t* chunk_offsets,
                                 msa_stream_t stream) {
  if (n_docs <= 0 || !tok_offsets || !chunk_offsets) return MSA_ERR_INVALID_ARG;
  if (chunk < 1 || chunk > msa::kMaxChunk) return MSA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  msa::chunk_offsets_kernel<<<1, 1024, 0, s>>>(n_docs, tok_offsets, chunk,
                                               chunk_offsets,
                                               msa::device_status_ptr());
  return msa::check_launch();
}

extern "C" int msa_encode_pool(msa_dtype dt, int L, int64_t n_tok, int n_docs,
                               int H, int D, const void* k_tok,
                               const void* v_tok, const void* kr_tok,
                               const int64_t* tok_offsets,
                               const int64_t* chunk_offsets, int64_t n_chunks,
                               float rope_base, int chunk, void* k_bar,
                               void* v_bar, void* kr_bar, msa_stream_t stream) {
  using namespace msa;
  if (L <= 0 || n_tok <= 0 || n_docs <= 0 || n_chunks < 0 || H <= 0) return MSA_ERR_INVALID_ARG;
  if (!k_tok || !v_tok || !kr_tok || !tok_offsets || !chunk_offsets || !k_bar ||
      !v_bar || !kr_bar)
    return MSA_ERR_INVALID_ARG;
  if (!aligned16(k_tok) || !aligned16(v_tok) || !aligned16(kr_tok) ||
      !aligned16(k_bar) || !aligned16(v_bar) || !aligned16(kr_bar))
    return MSA_ERR_INVALID_ARG;
  if (chunk < 1 || chunk > kMaxChunk || !(rope_base > 0.f)) return MSA_ERR_INVALID_ARG;
  if (H < 1 || H > 16 || (D != 64 && D != 128)) return MSA_ERR_UNSUPPORTED;
  if (n_chunks > 0x7fffffffLL) return MSA_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (dt == MSA_F32) {
    return D == 64 ? launch_encode<float, 64>(L, n_tok, n_docs, H, k_tok, v_tok, kr_tok,
                                              tok_offsets, chunk_offsets, n_chunks,
                                              rope_base, chunk, k_bar, v_bar, kr_bar, s)
                   : launch_encode<float, 128>(L, n_tok, n_docs, H, k_tok, v_tok, kr_tok,
                                               tok_offsets, chunk_offsets, n_chunks,
                                               rope_base, chunk, k_bar, v_bar, kr_bar, s);
  }
  if (dt == MSA_BF16) {
    return D == 64
               ? launch_encode<__nv_bfloat16, 64>(L, n_tok, n_docs, H, k_tok, v_tok, kr_tok,
                                                  tok_offsets, chunk_offsets, n_chunks,
                                                  rope_base, chunk, k_bar, v_bar, kr_bar, s)
               : launch_encode<__nv_bfloat16, 128>(L, n_tok, n_docs, H, k_tok, v_tok, kr_tok,
                                                   tok_offsets, chunk_offsets, n_chunks,
                                                   rope_base, chunk, k_bar, v_bar, kr_bar, s);
  }
  return MSA_ERR_INVALID_ARG;
}
