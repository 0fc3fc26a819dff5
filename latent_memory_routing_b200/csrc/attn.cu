// Sparse attention over [gathered memory rows ; local causal context], GQA,
// with global RoPE whose query start is offset by k.
//
// Method: "EverMind-AI/MSA: routing top-k compressed documents inside
// attention ..." (hysenlabs.com), §"Routing happens inside attention ..."
// (the top-k documents' compressed K/V are concatenated with the query's
// local K/V for autoregressive decoding) and §"Document-wise RoPE resets
// every document to position zero" (global RoPE: the query's starting index
// is offset by k, the number of retrieved blocks).  Readings: memory rows
// keep their document-wise rotation and are visible to every query token;
// local keys are causal; softmax scale 1/sqrt(D).
//
// This file holds the CUDA-core path for every fp32 call and the bf16 shapes
// the tensor-core prefill (attn_tc.cu) and the decode kernel
// (attn_decode.cu) do not take, and the entry point that picks among them
// by shape: a split-KV flash
// kernel -- one CTA per (query block, KV head, key split), 32-key tiles
// staged in shared memory in fp32 with local keys rotated on the way in,
// online softmax in fp32 per query row -- and the kernel that merges the
// splits.  The RoPE cos/sin of every local position is computed once per
// call (exact angle reduction in double) into the workspace.
#include <algorithm>
#include <cstdlib>

#include "attn_tc.cuh"
#include "msa_common.cuh"

namespace msa {
namespace {

constexpr int kAttnThreads = 128;
constexpr int kKeyTile = 32;
constexpr float kLog2e = 1.4426950408889634f;

struct AttnPlan {
  int G, TQ, ROWS, n_qblk, n_split;
  size_t cs_bytes, part_o_bytes, part_ml_bytes, total;
};

AttnPlan plan(int B, int T, int T_loc, int Hq, int H, int D, int m_cap, int sms) {
  AttnPlan p{};
  p.G = Hq / H;
  p.TQ = std::max(1, 16 / p.G);
  p.ROWS = p.G * p.TQ;
  p.n_qblk = (T + p.TQ - 1) / p.TQ;
  const int64_t base = (int64_t)B * H * p.n_qblk;
  const int64_t keys = (int64_t)m_cap + T_loc;
  int64_t ns = 1;
  if (base < 2LL * sms) ns = (2LL * sms + base - 1) / base;
  ns = std::min<int64_t>(ns, std::max<int64_t>(1, (keys + 63) / 64));
  ns = std::min<int64_t>(ns, 64);
  p.n_split = (int)ns;
  p.cs_bytes = round_up((size_t)T_loc * (D / 2) * sizeof(float2), 256);
  const size_t rows = (size_t)B * Hq * T;
  p.part_o_bytes = p.n_split > 1 ? round_up(rows * p.n_split * D * sizeof(float), 256) : 0;
  p.part_ml_bytes = p.n_split > 1 ? round_up(rows * p.n_split * sizeof(float2), 256) : 0;
  p.total = p.cs_bytes + p.part_o_bytes + p.part_ml_bytes;
  return p;
}

__global__ void rope_table_kernel(int n_pos, int half, int D, int64_t pos0, double base,
                                  float2* __restrict__ cs) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (int64_t)n_pos * half) return;
  const int j = (int)(e / half), i = (int)(e % half);
  cs[e] = rope_cs(pos0 + j, rope_inv_freq(base, i, D));
}

template <typename T, int D>
__global__ void __launch_bounds__(kAttnThreads)
attn_simt_kernel(int Tq, int T_loc, int Hq, int H, int G, int TQ, int ROWS,
                 const T* __restrict__ q, const T* __restrict__ k_mem,
                 const T* __restrict__ v_mem, const int32_t* __restrict__ mem_len, int m_cap,
                 const T* __restrict__ k_loc, const T* __restrict__ v_loc,
                 const float2* __restrict__ cs_tab, float qscale, int n_split,
                 T* __restrict__ out, float* __restrict__ part_o, float2* __restrict__ part_ml) {
  constexpr int HALF = D / 2;
  constexpr int PER = D / 32;
  constexpr int MAXR = 4;  // query rows per warp
  __shared__ float qs[16][D];
  __shared__ float ks[kKeyTile][D + 1];
  __shared__ float vs[kKeyTile][D];

  const int split = blockIdx.x, qblk = blockIdx.y;
  const int b = blockIdx.z / H, g = blockIdx.z % H;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int M = min(max(mem_len[b], 0), m_cap);
  const int tok0 = qblk * TQ;
  const int n_tok = min(TQ, Tq - tok0);
  const int rows = n_tok * G;

  // query rows: token tok0 + r / G, head g*G + r % G, rotated to its global
  // position pos0 + T_loc - Tq + token (cs_tab row T_loc - Tq + token)
  for (int e = tid; e < rows * HALF; e += kAttnThreads) {
    const int r = e / HALF, i = e % HALF;
    const int tok = tok0 + r / G, hq = g * G + r % G;
    const T* qp = q + (((int64_t)b * Tq + tok) * Hq + hq) * D;
    const float x1 = Elem<T>::to_f(qp[i]), x2 = Elem<T>::to_f(qp[i + HALF]);
    const float2 c = cs_tab[(int64_t)(T_loc - Tq + tok) * HALF + i];
    qs[r][i] = (x1 * c.x - x2 * c.y) * qscale;
    qs[r][i + HALF] = (x2 * c.x + x1 * c.y) * qscale;
  }

  // keys of this split; tokens of this block see local keys j <= lim_max
  const int n_keys = M + T_loc;
  const int chunk = (n_keys + n_split - 1) / n_split;
  const int k_lo = split * chunk;
  const int lim_max = T_loc - Tq + tok0 + n_tok - 1;
  const int k_hi = min(min(n_keys, k_lo + chunk), M + lim_max + 1);

  float m_run[MAXR], l_run[MAXR], o[MAXR][PER];
#pragma unroll
  for (int rr = 0; rr < MAXR; ++rr) {
    m_run[rr] = -INFINITY;
    l_run[rr] = 0.f;
#pragma unroll
    for (int x = 0; x < PER; ++x) o[rr][x] = 0.f;
  }
  __syncthreads();

  for (int t0 = k_lo; t0 < k_hi; t0 += kKeyTile) {
    for (int e = tid; e < kKeyTile * HALF; e += kAttnThreads) {
      const int j = e / HALF, i = e % HALF;
      const int kk = t0 + j;
      float k1 = 0.f, k2 = 0.f, v1 = 0.f, v2 = 0.f;
      if (kk < k_hi) {
        if (kk < M) {
          const int64_t off = (((int64_t)b * m_cap + kk) * H + g) * D;
          k1 = Elem<T>::to_f(k_mem[off + i]);
          k2 = Elem<T>::to_f(k_mem[off + i + HALF]);
          v1 = Elem<T>::to_f(v_mem[off + i]);
          v2 = Elem<T>::to_f(v_mem[off + i + HALF]);
        } else {
          const int jl = kk - M;
          const int64_t off = (((int64_t)b * T_loc + jl) * H + g) * D;
          const float x1 = Elem<T>::to_f(k_loc[off + i]);
          const float x2 = Elem<T>::to_f(k_loc[off + i + HALF]);
          const float2 c = cs_tab[(int64_t)jl * HALF + i];
          k1 = x1 * c.x - x2 * c.y;
          k2 = x2 * c.x + x1 * c.y;
          v1 = Elem<T>::to_f(v_loc[off + i]);
          v2 = Elem<T>::to_f(v_loc[off + i + HALF]);
        }
      }
      ks[j][i] = k1;
      ks[j][i + HALF] = k2;
      vs[j][i] = v1;
      vs[j][i + HALF] = v2;
    }
    __syncthreads();
    const int kk = t0 + lane;
#pragma unroll
    for (int rr = 0; rr < MAXR; ++rr) {
      const int r = warp + 4 * rr;
      if (r >= rows) break;  // warp-uniform
      float s = 0.f;
#pragma unroll 8
      for (int d = 0; d < D; ++d) s = fmaf(qs[r][d], ks[lane][d], s);
      const int tok = tok0 + r / G;
      const bool ok = kk < k_hi && (kk < M || kk - M <= T_loc - Tq + tok);
      s = ok ? s : -INFINITY;
      float mt = s;
#pragma unroll
      for (int off = 16; off; off >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
      const float m_new = fmaxf(m_run[rr], mt);
      if (m_new == -INFINITY) continue;  // nothing visible yet (warp-uniform)
      const float p = exp2f(s - m_new);
      const float corr = exp2f(m_run[rr] - m_new);
      float ps = p;
#pragma unroll
      for (int off = 16; off; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
      l_run[rr] = l_run[rr] * corr + ps;
      m_run[rr] = m_new;
#pragma unroll
      for (int x = 0; x < PER; ++x) o[rr][x] *= corr;
      for (int j = 0; j < kKeyTile; ++j) {
        const float pj = __shfl_sync(0xffffffffu, p, j);
#pragma unroll
        for (int x = 0; x < PER; ++x) o[rr][x] = fmaf(pj, vs[j][lane + 32 * x], o[rr][x]);
      }
    }
    __syncthreads();
  }

#pragma unroll
  for (int rr = 0; rr < MAXR; ++rr) {
    const int r = warp + 4 * rr;
    if (r >= rows) break;
    const int tok = tok0 + r / G, hq = g * G + r % G;
    const int64_t row_id = ((int64_t)b * Hq + hq) * Tq + tok;
    if (n_split == 1) {
      const float inv = l_run[rr] > 0.f ? 1.f / l_run[rr] : 0.f;
      T* op = out + (((int64_t)b * Tq + tok) * Hq + hq) * D;
#pragma unroll
      for (int x = 0; x < PER; ++x) op[lane + 32 * x] = Elem<T>::from_f(o[rr][x] * inv);
    } else {
      float* po = part_o + (row_id * n_split + split) * D;
#pragma unroll
      for (int x = 0; x < PER; ++x) po[lane + 32 * x] = o[rr][x];
      if (lane == 0) part_ml[row_id * n_split + split] = make_float2(m_run[rr], l_run[rr]);
    }
  }
}

// Merges the key splits of one (query, head, token) row.
template <typename T>
__global__ void attn_combine_kernel(int Tq, int Hq, int D, int n_split,
                                    const float* __restrict__ part_o,
                                    const float2* __restrict__ part_ml, T* __restrict__ out) {
  const int64_t row_id = blockIdx.x;  // ((b*Hq + hq)*Tq + tok)
  const int tok = (int)(row_id % Tq);
  const int hq = (int)((row_id / Tq) % Hq);
  const int64_t b = row_id / ((int64_t)Tq * Hq);
  const float2* ml = part_ml + row_id * n_split;
  float M = -INFINITY;
  for (int s = 0; s < n_split; ++s) M = fmaxf(M, ml[s].x);
  float L = 0.f;
  for (int s = 0; s < n_split; ++s)
    if (ml[s].x != -INFINITY) L += exp2f(ml[s].x - M) * ml[s].y;
  const float inv = L > 0.f ? 1.f / L : 0.f;
  T* op = out + ((b * Tq + tok) * Hq + hq) * D;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float acc = 0.f;
    for (int s = 0; s < n_split; ++s)
      if (ml[s].x != -INFINITY) acc += exp2f(ml[s].x - M) * part_o[(row_id * n_split + s) * D + d];
    op[d] = Elem<T>::from_f(acc * inv);
  }
}

}  // namespace

int attn_combine_bf16(int B, int T, int Hq, int D, int n_split, const float* part_o,
                      const float2* part_ml, void* out, cudaStream_t s) {
  attn_combine_kernel<__nv_bfloat16><<<(unsigned)((int64_t)B * Hq * T), 128, 0, s>>>(
      T, Hq, D, n_split, part_o, part_ml, static_cast<__nv_bfloat16*>(out));
  return check_launch();
}

namespace {

template <typename T, int D>
int launch_simt(int B, int Tq, int T_loc, int Hq, int H, const void* q, const void* k_mem,
                const void* v_mem, const int32_t* mem_len, int m_cap, const void* k_loc,
                const void* v_loc, const AttnPlan& p, const float2* cs, float qscale,
                float* part_o, float2* part_ml, void* out, cudaStream_t s) {
  const dim3 grid((unsigned)p.n_split, (unsigned)p.n_qblk, (unsigned)(B * H));
  attn_simt_kernel<T, D><<<grid, kAttnThreads, 0, s>>>(
      Tq, T_loc, Hq, H, p.G, p.TQ, p.ROWS, static_cast<const T*>(q),
      static_cast<const T*>(k_mem), static_cast<const T*>(v_mem), mem_len, m_cap,
      static_cast<const T*>(k_loc), static_cast<const T*>(v_loc), cs, qscale, p.n_split,
      static_cast<T*>(out), part_o, part_ml);
  int rc = check_launch();
  if (rc || p.n_split == 1) return rc;
  attn_combine_kernel<T><<<(unsigned)((int64_t)B * Hq * Tq), 128, 0, s>>>(
      Tq, Hq, D, p.n_split, part_o, part_ml, static_cast<T*>(out));
  return check_launch();
}

}  // namespace
}  // namespace msa

namespace msa {
namespace {
// bf16 decode runs on the tensor-core kernel unless MSA_DECODE_TC=0 selects
// the CUDA-core kernel (both compute the same attention)
bool decode_tc_enabled() {
  static const bool on = [] {
    const char* e = getenv("MSA_DECODE_TC");
    return !(e && e[0] == '0');
  }();
  return on;
}
}  // namespace
}  // namespace msa

extern "C" size_t msa_sparse_attn_workspace_size(msa_dtype dt, int B, int T, int T_loc, int Hq,
                                                 int H, int D, int m_cap) {
  using namespace msa;
  if (B <= 0 || T <= 0 || T_loc < T || H <= 0 || Hq % H || D <= 0 || m_cap < 0) return 0;
  if (dt == MSA_BF16 && attn_decode_supported(T, Hq, H, D))
    return std::max<size_t>({attn_decode_workspace_size(B, T_loc, Hq, H, D, m_cap),
                             attn_decode_tc_workspace_size(B, T_loc, Hq, H, D, m_cap),
                             (size_t)256});
  if (dt == MSA_BF16 && attn_tc_supported(B, T, T_loc, Hq, H, D, m_cap))
    return attn_tc_workspace_size(B, T, T_loc, Hq, H, D, m_cap);
  return plan(B, T, T_loc, Hq, H, D, m_cap, num_sms()).total;
}

static int sparse_attn_body(msa_dtype dt, int B, int T, int T_loc, int Hq, int H, int D,
                            const void* q, const void* k_mem, const void* v_mem,
                            const int32_t* mem_len, int m_cap, const void* k_loc,
                            const void* v_loc, int pos0, float rope_base, float scale,
                            void* out, void* ws, size_t ws_bytes, msa_stream_t stream) {
  using namespace msa;
  if (B <= 0 || T <= 0 || T_loc < T || H <= 0 || Hq <= 0 || m_cap < 0 || pos0 < 0)
    return MSA_ERR_INVALID_ARG;
  if (!q || !mem_len || !k_loc || !v_loc || !out) return MSA_ERR_INVALID_ARG;
  if (m_cap > 0 && (!k_mem || !v_mem)) return MSA_ERR_INVALID_ARG;
  if (!(rope_base > 0.f)) return MSA_ERR_INVALID_ARG;
  if (Hq % H || Hq / H > 16 || (D != 64 && D != 128)) return MSA_ERR_UNSUPPORTED;
  if (dt != MSA_F32 && dt != MSA_BF16) return MSA_ERR_INVALID_ARG;
  if ((int64_t)B * H > 65535 || (int64_t)m_cap + T_loc > (1LL << 30)) return MSA_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (int rc = debug_check_mem_len(mem_len, B, m_cap, s)) return rc;
  const float sc = scale > 0.f ? scale : 1.0f / sqrtf((float)D);
  const float qscale = sc * kLog2e;
  if (dt == MSA_BF16 && attn_decode_tc_supported(T, Hq, H, D) && decode_tc_enabled()) {
    const size_t need = attn_decode_tc_workspace_size(B, T_loc, Hq, H, D, m_cap);
    if (!ws || ws_bytes < need || !aligned16(ws)) return MSA_ERR_WORKSPACE;
    return attn_decode_tc_launch(B, T_loc, Hq, H, D, q, k_mem, v_mem, mem_len, m_cap, k_loc,
                                 v_loc, pos0, rope_base, qscale, out, ws, s);
  }
  if (dt == MSA_BF16 && attn_decode_supported(T, Hq, H, D)) {
    const size_t need = attn_decode_workspace_size(B, T_loc, Hq, H, D, m_cap);
    if (need && (!ws || ws_bytes < need || !aligned16(ws))) return MSA_ERR_WORKSPACE;
    return attn_decode_launch(B, T_loc, Hq, H, D, q, k_mem, v_mem, mem_len, m_cap, k_loc, v_loc,
                              pos0, rope_base, qscale, out, ws, s);
  }
  if (dt == MSA_BF16 && attn_tc_supported(B, T, T_loc, Hq, H, D, m_cap)) {
    const size_t need = attn_tc_workspace_size(B, T, T_loc, Hq, H, D, m_cap);
    if (!ws || ws_bytes < need || !aligned16(ws)) return MSA_ERR_WORKSPACE;
    return attn_tc_launch(B, T, T_loc, Hq, H, D, q, k_mem, v_mem, mem_len, m_cap, k_loc, v_loc,
                          pos0, rope_base, qscale, out, ws, s);
  }
  const AttnPlan p = plan(B, T, T_loc, Hq, H, D, m_cap, num_sms());
  if (!ws || ws_bytes < p.total || !aligned16(ws)) return MSA_ERR_WORKSPACE;
  unsigned char* w = static_cast<unsigned char*>(ws);
  float2* cs = reinterpret_cast<float2*>(w);
  float* part_o = reinterpret_cast<float*>(w + p.cs_bytes);
  float2* part_ml = reinterpret_cast<float2*>(w + p.cs_bytes + p.part_o_bytes);
  const int64_t n_cs = (int64_t)T_loc * (D / 2);
  rope_table_kernel<<<(unsigned)((n_cs + 255) / 256), 256, 0, s>>>(T_loc, D / 2, D, pos0,
                                                                  (double)rope_base, cs);
  int rc = check_launch();
  if (rc) return rc;
  if (dt == MSA_F32)
    return D == 64 ? launch_simt<float, 64>(B, T, T_loc, Hq, H, q, k_mem, v_mem, mem_len, m_cap,
                                            k_loc, v_loc, p, cs, qscale, part_o, part_ml, out, s)
                   : launch_simt<float, 128>(B, T, T_loc, Hq, H, q, k_mem, v_mem, mem_len, m_cap,
                                             k_loc, v_loc, p, cs, qscale, part_o, part_ml, out, s);
  return D == 64
             ? launch_simt<__nv_bfloat16, 64>(B, T, T_loc, Hq, H, q, k_mem, v_mem, mem_len, m_cap,
                                              k_loc, v_loc, p, cs, qscale, part_o, part_ml, out, s)
             : launch_simt<__nv_bfloat16, 128>(B, T, T_loc, Hq, H, q, k_mem, v_mem, mem_len,
                                               m_cap, k_loc, v_loc, p, cs, qscale, part_o,
                                               part_ml, out, s);
}

extern "C" int msa_sparse_attn(msa_dtype dt, int B, int T, int T_loc, int Hq, int H, int D,
                               const void* q, const void* k_mem, const void* v_mem,
                               const int32_t* mem_len, int m_cap, const void* k_loc,
                               const void* v_loc, int pos0, float rope_base, float scale,
                               void* out, void* ws, size_t ws_bytes, msa_stream_t stream) {
  return msa::debug_finish(sparse_attn_body(dt, B, T, T_loc, Hq, H, D, q, k_mem, v_mem, mem_len,
                                            m_cap, k_loc, v_loc, pos0, rope_base, scale, out,
                                            ws, ws_bytes, stream),
                           reinterpret_cast<cudaStream_t>(stream));
}
