// Backward pass of chunk pooling and routing, for training with a routing
// loss.
//
// Method: "深度分析MSA:把超长文档组织成可检索内部记忆的工程路径"
// (yeyulingfeng.com), §"四、训练阶段：学习 memory 与路由": a training step
// pools the documents' token K/V/K_r into the memory, routes Q_r against the
// pooled routing keys, and the routing auxiliary loss (BCE or InfoNCE on the
// document scores) sends gradients back to Q_r and, through the pooling, to
// the token-level K_r.  The loss is the caller's; these kernels turn
// dL/d(document scores) into dL/dQ_r and dL/dK̄_r, and dL/d(pooled bank)
// into dL/d(token tensors).
//
// Readings (where the page is silent): the gradient of a maximum goes to its
// first maximiser -- a document's best (chunk, query token) pair, the lowest
// chunk and then the lowest token among equals; each cosine norm is
// max(|x|, 1e-12), a constant below 1e-12; the pooling backward is the
// pooling's adjoint (K's gradient rotated back by the token's document-wise
// position).
//
// Design.
//  * pool_backward_kernel: one CTA per chunk (like the forward), the chunk's
//    (cos, sin) table built once (angles reduced in double); every token row
//    of every layer is written once with 16-byte stores: V and K_r get the
//    pooled gradient / count, K its rotation by -p.  HBM-bound on the writes.
//  * routing, bf16 (the tensor-core path): finding each document's first
//    maximiser is the forward scan itself -- every (chunk, token) head-mean
//    cosine -- so it runs as the tcgen05 routing kernel in its argmax mode
//    (one 64-bit key per (query, document): score, then ~(chunk, token));
//    route_grad_kernel then takes one warp per pair with a non-zero gradient
//    and adds g/H * dcos/dq and g/H * dcos/dk for each head into dq_r and
//    dkr_bar (fp32, atomically: pairs may share a token or a chunk).  The
//    maximiser is decided on the scan's bf16 unit rows (fp32 sums); the
//    gradient is taken from the inputs in fp32.
//  * routing, fp32 (or MSA_ROUTE_BWD_TC=0): route_backward_kernel,
//    persistent CTAs over the pairs with a non-zero gradient, recomputes the
//    document's cosines in fp32 on the CUDA cores from unit rows staged in
//    shared memory (8 chunks x 16 tokens at a time, two threads per pair),
//    takes the first maximiser and adds the same gradients.  Its cost grows
//    with the pairs that carry gradient, not with the bank.
#include <algorithm>

#include <cstdlib>

#include "msa_common.cuh"
#include "route_tc.cuh"

namespace msa {
namespace {

constexpr int kPbThreads = 256;
constexpr int kChunkTok = 64;

template <int D>
__global__ void __launch_bounds__(kPbThreads)
pool_backward_kernel(int L, int64_t n_tok, int n_docs, int H,
                     const float* __restrict__ dk_bar, const float* __restrict__ dv_bar,
                     const float* __restrict__ dkr_bar, const int64_t* __restrict__ tok_off,
                     const int64_t* __restrict__ chunk_off, int64_t n_chunks, double base,
                     float* __restrict__ dk_tok, float* __restrict__ dv_tok,
                     float* __restrict__ dkr_tok) {
  constexpr int HALF = D / 2;
  __shared__ float2 cs_tab[kChunkTok][HALF];  // (cos, sin) of p * w_i
  __shared__ double w_tab[HALF];
  __shared__ int64_t s_tok0, s_p0;
  __shared__ int s_rows;
  const int tid = threadIdx.x;
  const int64_t c = blockIdx.x;
  if (tid < 32) {
    const int64_t d = warp_find_segment(chunk_off, n_docs, c);
    if (tid == 0) {
      const int64_t j = c - chunk_off[d];
      const int64_t t0 = tok_off[d] + j * kChunkTok;
      const int64_t left = tok_off[d + 1] - t0;
      s_tok0 = t0;
      s_p0 = j * kChunkTok;
      s_rows = (int)(left < 0 ? 0 : (left < kChunkTok ? left : kChunkTok));
    }
  }
  for (int i = tid; i < HALF; i += blockDim.x) w_tab[i] = rope_inv_freq(base, i, D);
  __syncthreads();
  const int rows = s_rows;
  const int64_t tok0 = s_tok0, p0 = s_p0;
  for (int e = tid; e < rows * HALF; e += blockDim.x)
    cs_tab[e / HALF][e % HALF] = rope_cs(p0 + e / HALF, w_tab[e % HALF]);
  __syncthreads();
  if (rows == 0) return;
  const float inv_n = 1.0f / (float)rows;
  const int64_t row_elems = (int64_t)H * D;
  const int UPH = HALF / 4;  // float4 pair-vectors per head
  for (int l = 0; l < L; ++l) {
    const float* gk = dk_bar + ((int64_t)l * n_chunks + c) * row_elems;
    const float* gv = dv_bar + ((int64_t)l * n_chunks + c) * row_elems;
    const float* gr = dkr_bar + ((int64_t)l * n_chunks + c) * row_elems;
    const int64_t out0 = ((int64_t)l * n_tok + tok0) * row_elems;
    // V and K_r: the pooled gradient / count on every token of the chunk
    for (int e = tid; e < rows * (int)(row_elems / 4); e += blockDim.x) {
      const int t = e / (int)(row_elems / 4), col = (e % (int)(row_elems / 4)) * 4;
      const float4 a = *reinterpret_cast<const float4*>(gv + col);
      const float4 bb = *reinterpret_cast<const float4*>(gr + col);
      *reinterpret_cast<float4*>(dv_tok + out0 + t * row_elems + col) =
          make_float4(a.x * inv_n, a.y * inv_n, a.z * inv_n, a.w * inv_n);
      *reinterpret_cast<float4*>(dkr_tok + out0 + t * row_elems + col) =
          make_float4(bb.x * inv_n, bb.y * inv_n, bb.z * inv_n, bb.w * inv_n);
    }
    // K: rotated back by -p, pair (i, i + D/2), four pairs per thread
    for (int e = tid; e < rows * H * UPH; e += blockDim.x) {
      const int t = e / (H * UPH), h = (e / UPH) % H, v = e % UPH;
      const int col = h * D + v * 4;
      const float4 x1 = *reinterpret_cast<const float4*>(gk + col);
      const float4 x2 = *reinterpret_cast<const float4*>(gk + col + HALF);
      const float a1[4] = {x1.x, x1.y, x1.z, x1.w}, a2[4] = {x2.x, x2.y, x2.z, x2.w};
      float y1[4], y2[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 q = cs_tab[t][v * 4 + i];
        y1[i] = (a1[i] * q.x + a2[i] * q.y) * inv_n;  // R(-p): sin -> -sin
        y2[i] = (a2[i] * q.x - a1[i] * q.y) * inv_n;
      }
      float* o = dk_tok + out0 + t * row_elems + col;
      *reinterpret_cast<float4*>(o) = make_float4(y1[0], y1[1], y1[2], y1[3]);
      *reinterpret_cast<float4*>(o + HALF) = make_float4(y2[0], y2[1], y2[2], y2[3]);
    }
  }
}

constexpr int kRbThreads = 256;
constexpr int kRbChunks = 8;   // chunks staged at a time
constexpr int kRbTokens = 16;  // query tokens staged at a time
constexpr float kEps = 1e-12f;

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}

// Lexicographic "better" for the first maximiser: higher score, then lower
// chunk, then lower token.
__device__ __forceinline__ bool better(float s, int c, int t, float s2, int c2, int t2) {
  if (s != s2) return s > s2;
  if (c != c2) return c < c2;
  return t < t2;
}

// Stages `n` rows of H x D (each a (row, head) vector of D elements) as unit
// vectors (x / max(|x|, eps)) in fp32: one warp per (row, head) vector.
template <typename T>
__device__ void stage_unit_rows(const T* __restrict__ src, int64_t row_stride, int n, int H,
                                int D, float* dst) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int v = warp; v < n * H; v += kRbThreads / 32) {
    const int r = v / H, h = v % H;
    const T* x = src + r * row_stride + h * D;
    float ss = 0.f;
    for (int i = lane; i < D; i += 32) {
      const float f = to_f(x[i]);
      ss = fmaf(f, f, ss);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float inv = 1.0f / fmaxf(sqrtf(ss), kEps);
    for (int i = lane; i < D; i += 32) dst[(r * H + h) * D + i] = to_f(x[i]) * inv;
  }
}

template <typename E>
__global__ void __launch_bounds__(kRbThreads)
route_backward_kernel(int B, int T, int H, int D, const E* __restrict__ q_r,
                      const E* __restrict__ kr, const int64_t* __restrict__ coff, int n_docs,
                      const float* __restrict__ d_doc, float* __restrict__ dq,
                      float* __restrict__ dkr, int* status) {
  extern __shared__ __align__(16) float rb_smem[];
  float* kh = rb_smem;                            // [kRbChunks][H][D] unit rows
  float* qh = kh + kRbChunks * H * D;             // [kRbTokens][H][D] unit rows
  __shared__ float s_best[kRbThreads / 32];
  __shared__ int s_bc[kRbThreads / 32], s_bt[kRbThreads / 32];
  __shared__ float s_nq[16], s_nk[16], s_dot[16];
  __shared__ int s_c, s_t;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t HD = (int64_t)H * D;
  const int64_t n_pairs = (int64_t)B * n_docs;
  for (int64_t pr = blockIdx.x; pr < n_pairs; pr += gridDim.x) {
    const float g = d_doc[pr];
    if (g == 0.f) continue;  // uniform over the CTA
    const int b = (int)(pr / n_docs), d = (int)(pr % n_docs);
    const int64_t c0 = coff[d], c1 = coff[d + 1];
    if (c1 <= c0) {
      if (tid == 0) record_error(status, MSA_ERR_INVALID_ARG);
      continue;
    }
    // ---- first maximiser of the head-mean cosine over (chunk, token)
    float best = -INFINITY;
    int bc = INT32_MAX, bt = INT32_MAX;
    const int pair = tid >> 1, half = tid & 1;  // two threads per (chunk, token)
    const int pc = pair / kRbTokens, pt = pair % kRbTokens;
    for (int64_t cg = c0; cg < c1; cg += kRbChunks) {
      const int nc = (int)(c1 - cg < kRbChunks ? c1 - cg : kRbChunks);
      __syncthreads();  // kh is about to be rewritten
      stage_unit_rows(kr + cg * HD, HD, nc, H, D, kh);
      for (int t0 = 0; t0 < T; t0 += kRbTokens) {
        const int ntk = min(kRbTokens, T - t0);
        __syncthreads();  // qh is about to be rewritten (and kh is ready)
        stage_unit_rows(q_r + ((int64_t)b * T + t0) * HD, HD, ntk, H, D, qh);
        __syncthreads();
        float s = 0.f;
        if (pc < nc && pt < ntk) {
          for (int h = half; h < H; h += 2) {
            const float4* a = reinterpret_cast<const float4*>(kh + (pc * H + h) * D);
            const float4* bq = reinterpret_cast<const float4*>(qh + (pt * H + h) * D);
            for (int i = 0; i < D / 4; ++i) {
              const float4 x = a[i], y = bq[i];
              s = fmaf(x.x, y.x, s);
              s = fmaf(x.y, y.y, s);
              s = fmaf(x.z, y.z, s);
              s = fmaf(x.w, y.w, s);
            }
          }
        }
        s += __shfl_xor_sync(0xffffffffu, s, 1);
        if (half == 0 && pc < nc && pt < ntk) {
          const float sc = s / (float)H;
          const int c = (int)(cg + pc), t = t0 + pt;
          if (better(sc, c, t, best, bc, bt)) {
            best = sc;
            bc = c;
            bt = t;
          }
        }
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      const float s2 = __shfl_xor_sync(0xffffffffu, best, o);
      const int c2 = __shfl_xor_sync(0xffffffffu, bc, o), t2 = __shfl_xor_sync(0xffffffffu, bt, o);
      if (better(s2, c2, t2, best, bc, bt)) {
        best = s2;
        bc = c2;
        bt = t2;
      }
    }
    if (lane == 0) {
      s_best[warp] = best;
      s_bc[warp] = bc;
      s_bt[warp] = bt;
    }
    __syncthreads();
    if (tid == 0) {
      float bs = s_best[0];
      int cc = s_bc[0], tt = s_bt[0];
      for (int w = 1; w < kRbThreads / 32; ++w)
        if (better(s_best[w], s_bc[w], s_bt[w], bs, cc, tt)) {
          bs = s_best[w];
          cc = s_bc[w];
          tt = s_bt[w];
        }
      s_c = cc;
      s_t = tt;
    }
    __syncthreads();
    const int cs = s_c, ts = s_t;
    // ---- gradients of (1/H) sum_h cos(q_h, k_h) at (token ts, chunk cs)
    const E* qv = q_r + ((int64_t)b * T + ts) * HD;
    const E* kv = kr + (int64_t)cs * HD;
    for (int h = warp; h < H; h += kRbThreads / 32) {
      float nq = 0.f, nk = 0.f, dt = 0.f;
      for (int i = lane; i < D; i += 32) {
        const float x = to_f(qv[h * D + i]), y = to_f(kv[h * D + i]);
        nq = fmaf(x, x, nq);
        nk = fmaf(y, y, nk);
        dt = fmaf(x, y, dt);
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) {
        nq += __shfl_xor_sync(0xffffffffu, nq, o);
        nk += __shfl_xor_sync(0xffffffffu, nk, o);
        dt += __shfl_xor_sync(0xffffffffu, dt, o);
      }
      if (lane == 0) {
        s_nq[h] = sqrtf(nq);
        s_nk[h] = sqrtf(nk);
        s_dot[h] = dt;
      }
    }
    __syncthreads();
    const float gh = g / (float)H;
    for (int e = tid; e < (int)HD; e += blockDim.x) {
      const int h = e / D;
      const float lq = s_nq[h], lk = s_nk[h];
      const float mq = fmaxf(lq, kEps), mk = fmaxf(lk, kEps);
      const float cosv = s_dot[h] / (mq * mk);
      const float x = to_f(qv[e]), y = to_f(kv[e]);
      const float gq = y / (mq * mk) - (lq >= kEps ? cosv * x / (mq * mq) : 0.f);
      const float gk = x / (mq * mk) - (lk >= kEps ? cosv * y / (mk * mk) : 0.f);
      atomicAdd(dq + ((int64_t)b * T + ts) * HD + e, gh * gq);
      atomicAdd(dkr + (int64_t)cs * HD + e, gh * gk);
    }
  }
}

// Gradients at known first maximisers (the tensor-core argmax scan's keys):
// one warp per (query, document) pair with a non-zero gradient; per head the
// warp reduces |q|, |k| and q.k over D and adds g/H * dcos/dq and
// g/H * dcos/dk into dq_r and dkr_bar.
template <typename E>
__global__ void __launch_bounds__(256)
route_grad_kernel(int B, int T, int H, int D, const E* __restrict__ q_r,
                  const E* __restrict__ kr, const int64_t* __restrict__ coff, int n_docs,
                  const float* __restrict__ d_doc, const unsigned long long* __restrict__ keys,
                  float* __restrict__ dq, float* __restrict__ dkr, int* status) {
  const int lane = threadIdx.x & 31;
  const int64_t HD = (int64_t)H * D;
  const int64_t n_pairs = (int64_t)B * n_docs;
  const int64_t w0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t pr = w0; pr < n_pairs; pr += nw) {
    const float g = d_doc[pr];
    if (g == 0.f) continue;
    const unsigned long long key = keys[pr];
    if (key == 0ull) {  // no chunk reached this pair (an empty document)
      if (lane == 0) record_error(status, MSA_ERR_INVALID_ARG);
      continue;
    }
    const int b = (int)(pr / n_docs), d = (int)(pr % n_docs);
    const uint32_t local = 0xffffffffu - (uint32_t)key;
    const int64_t cs = coff[d] + local / (uint32_t)T;
    const int ts = (int)(local % (uint32_t)T);
    const E* qv = q_r + ((int64_t)b * T + ts) * HD;
    const E* kv = kr + cs * HD;
    float* gq_out = dq + ((int64_t)b * T + ts) * HD;
    float* gk_out = dkr + cs * HD;
    const float gh = g / (float)H;
    for (int h = 0; h < H; ++h) {
      float nq = 0.f, nk = 0.f, dt = 0.f;
      for (int i = lane; i < D; i += 32) {
        const float x = to_f(qv[h * D + i]), y = to_f(kv[h * D + i]);
        nq = fmaf(x, x, nq);
        nk = fmaf(y, y, nk);
        dt = fmaf(x, y, dt);
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) {
        nq += __shfl_xor_sync(0xffffffffu, nq, o);
        nk += __shfl_xor_sync(0xffffffffu, nk, o);
        dt += __shfl_xor_sync(0xffffffffu, dt, o);
      }
      const float lq = sqrtf(nq), lk = sqrtf(nk);
      const float mq = fmaxf(lq, kEps), mk = fmaxf(lk, kEps);
      const float cosv = dt / (mq * mk);
      for (int i = lane; i < D; i += 32) {
        const float x = to_f(qv[h * D + i]), y = to_f(kv[h * D + i]);
        const float gq = y / (mq * mk) - (lq >= kEps ? cosv * x / (mq * mq) : 0.f);
        const float gk = x / (mq * mk) - (lk >= kEps ? cosv * y / (mk * mk) : 0.f);
        atomicAdd(gq_out + h * D + i, gh * gq);
        atomicAdd(gk_out + h * D + i, gh * gk);
      }
    }
  }
}

// The tensor-core path: bf16, D in {64, 128}, H <= 8, and every document's
// (chunk, token) index fits the key's 32 bits (bounded by n_chunks * T).
bool route_backward_tc(msa_dtype dt, int B, int T, int H, int D, int64_t n_chunks) {
  static const bool enabled = [] {
    const char* e = getenv("MSA_ROUTE_BWD_TC");
    return !(e && e[0] == '0');
  }();
  return enabled && dt == MSA_BF16 && (D == 64 || D == 128) && H <= 8 &&
         (int64_t)B * T <= (1LL << 24) && n_chunks * (int64_t)T < 0xffffffffLL;
}

struct BwdPlan {
  int n_pad;
  size_t q_bytes, key_bytes, total;
};

BwdPlan bwd_plan(int B, int T, int H, int D, int n_docs) {
  BwdPlan p{};
  p.n_pad = (int)route_tc_columns((int64_t)B * T);
  p.q_bytes = round_up((size_t)p.n_pad * H * D * sizeof(__nv_bfloat16), 256);
  p.key_bytes = round_up((size_t)B * n_docs * sizeof(unsigned long long), 256);
  p.total = p.q_bytes + p.key_bytes;
  return p;
}

}  // namespace
}  // namespace msa

extern "C" size_t msa_route_backward_workspace_size(msa_dtype dt, int B, int T, int H, int D,
                                                    int64_t n_chunks, int n_docs) {
  using namespace msa;
  if (B <= 0 || T <= 0 || H <= 0 || n_docs <= 0 || n_chunks <= 0) return 0;
  if (!route_backward_tc(dt, B, T, H, D, n_chunks)) return 0;
  return bwd_plan(B, T, H, D, n_docs).total;
}

extern "C" int msa_encode_pool_backward(int L, int64_t n_tok, int n_docs, int H, int D,
                                        const float* dk_bar, const float* dv_bar,
                                        const float* dkr_bar, const int64_t* tok_offsets,
                                        const int64_t* chunk_offsets, int64_t n_chunks,
                                        float rope_base, float* dk_tok, float* dv_tok,
                                        float* dkr_tok, msa_stream_t stream) {
  using namespace msa;
  if (L <= 0 || n_tok <= 0 || n_docs <= 0 || H <= 0 || n_chunks <= 0) return MSA_ERR_INVALID_ARG;
  if (!dk_bar || !dv_bar || !dkr_bar || !tok_offsets || !chunk_offsets || !dk_tok || !dv_tok ||
      !dkr_tok)
    return MSA_ERR_INVALID_ARG;
  if (!(rope_base > 0.f)) return MSA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return MSA_ERR_UNSUPPORTED;
  if (!aligned16(dk_bar) || !aligned16(dv_bar) || !aligned16(dkr_bar) || !aligned16(dk_tok) ||
      !aligned16(dv_tok) || !aligned16(dkr_tok))
    return MSA_ERR_INVALID_ARG;
  if (n_chunks > 0x7fffffffLL) return MSA_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (int rc = debug_check_offsets(tok_offsets, n_docs, n_tok, s)) return rc;
  if (int rc = debug_check_offsets(chunk_offsets, n_docs, n_chunks, s)) return rc;
  if (D == 64)
    pool_backward_kernel<64><<<(unsigned)n_chunks, kPbThreads, 0, s>>>(
        L, n_tok, n_docs, H, dk_bar, dv_bar, dkr_bar, tok_offsets, chunk_offsets, n_chunks,
        (double)rope_base, dk_tok, dv_tok, dkr_tok);
  else
    pool_backward_kernel<128><<<(unsigned)n_chunks, kPbThreads, 0, s>>>(
        L, n_tok, n_docs, H, dk_bar, dv_bar, dkr_bar, tok_offsets, chunk_offsets, n_chunks,
        (double)rope_base, dk_tok, dv_tok, dkr_tok);
  return debug_finish(check_launch(), s);
}

extern "C" int msa_route_backward(msa_dtype dt, int B, int T, int H, int D, const void* q_r,
                                  const void* kr_bar, int64_t n_chunks,
                                  const int64_t* chunk_offsets, int n_docs, const float* d_doc,
                                  float* dq_r, float* dkr_bar, void* ws, size_t ws_bytes,
                                  msa_stream_t stream) {
  using namespace msa;
  if (B <= 0 || T <= 0 || H <= 0 || D <= 0 || n_chunks <= 0 || n_docs <= 0)
    return MSA_ERR_INVALID_ARG;
  if (!q_r || !kr_bar || !chunk_offsets || !d_doc || !dq_r || !dkr_bar) return MSA_ERR_INVALID_ARG;
  if ((D != 64 && D != 128) || H > 16 || (int64_t)H * D > 1024) return MSA_ERR_UNSUPPORTED;
  if (dt != MSA_F32 && dt != MSA_BF16) return MSA_ERR_INVALID_ARG;
  if (n_chunks > 0x7fffffffLL || (int64_t)B * T > 0x7fffffffLL) return MSA_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (int rc = debug_check_offsets(chunk_offsets, n_docs, n_chunks, s)) return rc;
  if (route_backward_tc(dt, B, T, H, D, n_chunks)) {
    // (1) the first maximiser of every (query, document) on the tensor
    // cores; (2) the cosine gradients at those pairs on the CUDA cores
    const BwdPlan p = bwd_plan(B, T, H, D, n_docs);
    if (!ws || ws_bytes < p.total || !aligned16(ws)) return MSA_ERR_WORKSPACE;
    if (!aligned16(q_r) || !aligned16(kr_bar)) return MSA_ERR_INVALID_ARG;
    unsigned char* w = static_cast<unsigned char*>(ws);
    auto* qhat = reinterpret_cast<__nv_bfloat16*>(w);
    auto* keys = reinterpret_cast<unsigned long long*>(w + p.q_bytes);
    const auto* q = static_cast<const __nv_bfloat16*>(q_r);
    const auto* k = static_cast<const __nv_bfloat16*>(kr_bar);
    int rc = route_prep_bf16_launch(B * T, H, D, p.n_pad, q, qhat, s);
    if (rc) return rc;
    if ((rc = note_cuda(cudaMemsetAsync(keys, 0, (size_t)B * n_docs * 8, s)))) return rc;
    rc = route_tc_argmax_launch(B, T, H, D, qhat, p.n_pad, k, n_chunks, chunk_offsets, n_docs,
                                keys, device_status_ptr(), s);
    if (rc) return rc;
    const int64_t pairs = (int64_t)B * n_docs;
    const int grid = (int)std::min<int64_t>((pairs + 7) / 8, 16LL * num_sms());
    route_grad_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(B, T, H, D, q, k, chunk_offsets, n_docs,
                                                          d_doc, keys, dq_r, dkr_bar,
                                                          device_status_ptr());
    return debug_finish(check_launch(), s);
  }
  const size_t smem = (size_t)(kRbChunks + kRbTokens) * H * D * sizeof(float);
  const int64_t pairs = (int64_t)B * n_docs;
  const int grid = (int)std::min<int64_t>(pairs, 8LL * num_sms());
  if (dt == MSA_F32) {
    auto k = route_backward_kernel<float>;
    int rc = ensure_smem_attr(reinterpret_cast<const void*>(k), (int)smem);
    if (rc) return rc;
    k<<<grid, kRbThreads, smem, s>>>(B, T, H, D, static_cast<const float*>(q_r),
                                     static_cast<const float*>(kr_bar), chunk_offsets, n_docs,
                                     d_doc, dq_r, dkr_bar, device_status_ptr());
  } else {
    auto k = route_backward_kernel<__nv_bfloat16>;
    int rc = ensure_smem_attr(reinterpret_cast<const void*>(k), (int)smem);
    if (rc) return rc;
    k<<<grid, kRbThreads, smem, s>>>(B, T, H, D, static_cast<const __nv_bfloat16*>(q_r),
                                     static_cast<const __nv_bfloat16*>(kr_bar), chunk_offsets,
                                     n_docs, d_doc, dq_r, dkr_bar, device_status_ptr());
  }
  return debug_finish(check_launch(), s);
}
