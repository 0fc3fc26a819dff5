// bf16 decode attention (one query token) over [gathered memory ; local
// context], GQA, global RoPE offset by k.
//
// Method: "EverMind-AI/MSA: routing top-k compressed documents inside
// attention ..." (hysenlabs.com), §"Routing happens inside attention ..."
// (the selected documents' compressed K/V are concatenated with the query's
// local K/V for autoregressive decoding) and §"Document-wise RoPE resets
// every document to position zero" (global RoPE, query start offset by k).
// The query is the last of the T_loc local tokens and sees every key.
//
// Design (HBM-bound: every K/V byte is read once).  One CTA of 128 threads
// per (key split, batch element, KV head), serving the G query heads that
// share the KV head:
//   * 64-key tiles of K and V are streamed with 16-byte cp.async into a
//     2-stage shared ring (64 KB + 32 KB of RoPE state: two CTAs per SM);
//   * two threads per key row each own half of the rotate-half pairs; a
//     local row is rotated in registers with (cos, sin) of its position held
//     in shared memory for the tile's 64 rows -- anchored exactly (angles
//     reduced in double) at the CTA's first local tile and advanced by one
//     complex multiply per tile (the rows move 64 positions), so drift stays
//     at a few 1e-7 over a split -- then dotted with the G rotated queries;
//   * one warp per query head runs the online softmax over the tile and
//     accumulates O (4 dims per lane) from the V tile;
//   * splits write (max, sum, O) partials that the split-KV combine kernel
//     merges; a single split writes the normalised output directly.
#include <algorithm>

#include "attn_tc.cuh"
#include "msa_common.cuh"

namespace msa {
namespace {

constexpr int kDThreads = 128;
constexpr int kDKeys = 64;  // keys per tile
constexpr int kDStages = 2;

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(smem))),
               "l"(gmem)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int D, int G>
__global__ void __launch_bounds__(kDThreads, 2)
attn_decode_kernel(int T_loc, int Hq, int H, const __nv_bfloat16* __restrict__ q,
                   const __nv_bfloat16* __restrict__ k_mem,
                   const __nv_bfloat16* __restrict__ v_mem, const int32_t* __restrict__ mem_len,
                   int m_cap, const __nv_bfloat16* __restrict__ k_loc,
                   const __nv_bfloat16* __restrict__ v_loc, int64_t pos0, double base,
                   float qscale, int n_split, __nv_bfloat16* __restrict__ out,
                   float* __restrict__ part_o, float2* __restrict__ part_ml) {
  constexpr int HALF = D / 2;
  constexpr int QP = HALF / 2;            // pairs per thread (two threads per row)
  constexpr int ROW_B = D * 2;            // bytes per K/V row
  constexpr int VPL = D / 32;             // output dims per lane
  extern __shared__ __align__(16) unsigned char smem[];
  unsigned char* sK = smem;                                        // [stage][64][D] bf16
  unsigned char* sV = sK + kDStages * kDKeys * ROW_B;              // [stage][64][D] bf16
  float2* cs = reinterpret_cast<float2*>(sV + kDStages * kDKeys * ROW_B);  // [64][HALF]
  static_assert(D == 128, "four output dims per lane");
  __shared__ float2 step[HALF];                   // e^{i 64 w_i}
  __shared__ __align__(16) float qs[G][D];        // rotated, scaled queries
  __shared__ float sc[G][kDKeys];                 // tile scores, then probabilities
  __shared__ double wf[HALF];                     // inverse frequencies

  const int split = blockIdx.x;
  const int b = blockIdx.y / H, g = blockIdx.y % H;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int M = min(max(mem_len[b], 0), m_cap);
  const int n_keys = M + T_loc;
  const int per = (n_keys + n_split - 1) / n_split;
  const int k_lo = min(n_keys, split * per), k_hi = min(n_keys, k_lo + per);
  const int n_tiles = (k_hi - k_lo + kDKeys - 1) / kDKeys;

  for (int i = tid; i < HALF; i += kDThreads) wf[i] = rope_inv_freq(base, i, D);
  __syncthreads();
  // queries of the group, rotated to pos0 + T_loc - 1 and scaled
  for (int e = tid; e < G * HALF; e += kDThreads) {
    const int h = e / HALF, i = e % HALF;
    const __nv_bfloat16* qp = q + ((int64_t)b * Hq + g * G + h) * D;
    const float x1 = __bfloat162float(qp[i]), x2 = __bfloat162float(qp[i + HALF]);
    const float2 c = rope_cs(pos0 + T_loc - 1, wf[i]);
    qs[h][i] = (x1 * c.x - x2 * c.y) * qscale;
    qs[h][i + HALF] = (x2 * c.x + x1 * c.y) * qscale;
  }
  for (int i = tid; i < HALF; i += kDThreads) step[i] = rope_cs(kDKeys, wf[i]);

  auto load_tile = [&](int t, int st) {
    const int key0 = k_lo + t * kDKeys;
    for (int c = tid; c < kDKeys * (ROW_B / 16); c += kDThreads) {
      const int r = c / (ROW_B / 16), piece = c % (ROW_B / 16);
      const int key = key0 + r;
      unsigned char* kd = sK + (st * kDKeys + r) * ROW_B + piece * 16;
      unsigned char* vd = sV + (st * kDKeys + r) * ROW_B + piece * 16;
      if (key < k_hi) {
        const __nv_bfloat16 *ks, *vs;
        if (key < M) {
          const int64_t off = (((int64_t)b * m_cap + key) * H + g) * D + piece * 8;
          ks = k_mem + off;
          vs = v_mem + off;
        } else {
          const int64_t off = (((int64_t)b * T_loc + key - M) * H + g) * D + piece * 8;
          ks = k_loc + off;
          vs = v_loc + off;
        }
        cp_async16(kd, ks);
        cp_async16(vd, vs);
      } else {
        *reinterpret_cast<uint4*>(kd) = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(vd) = make_uint4(0, 0, 0, 0);
      }
    }
    cp_async_commit();
  };

  // running softmax state: warp w owns heads w, w+4, ...
  constexpr int HPW = (G + 3) / 4;
  float m_run[HPW], l_run[HPW], o[HPW][VPL];
#pragma unroll
  for (int a = 0; a < HPW; ++a) {
    m_run[a] = -INFINITY;
    l_run[a] = 0.f;
#pragma unroll
    for (int x = 0; x < VPL; ++x) o[a][x] = 0.f;
  }

  const int row = tid >> 1, hp = tid & 1;  // key row and pair half of this thread
  bool cs_ready = false;
  if (n_tiles > 0) load_tile(0, 0);
  for (int t = 0; t < n_tiles; ++t) {
    const int st = t & 1;
    const int key0 = k_lo + t * kDKeys;
    if (t + 1 < n_tiles) {
      load_tile(t + 1, st ^ 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    // (cos, sin) of this tile's rows: anchored at the first tile holding a
    // local row, then advanced by 64 positions per tile
    const bool any_local = key0 + kDKeys > M;
    if (any_local && !cs_ready) {
      for (int e = tid; e < kDKeys * HALF; e += kDThreads) {
        const int r = e / HALF, i = e % HALF;
        cs[e] = rope_cs(pos0 + (int64_t)(key0 + r - M), wf[i]);
      }
      cs_ready = true;
    } else if (any_local) {
      for (int e = tid; e < kDKeys * HALF; e += kDThreads) {
        const float2 a = cs[e], w = step[e % HALF];
        cs[e] = make_float2(a.x * w.x - a.y * w.y, a.x * w.y + a.y * w.x);
      }
    }
    __syncthreads();

    // scores of (row, head) -- two threads per row, HALF/2 pairs each
    {
      const unsigned char* kr = sK + (st * kDKeys + row) * ROW_B;
      const bool local = key0 + row >= M;
      float acc[G];
#pragma unroll
      for (int h = 0; h < G; ++h) acc[h] = 0.f;
#pragma unroll
      for (int v8 = 0; v8 < QP / 8; ++v8) {
        const int i0 = hp * QP + v8 * 8;  // first pair index of this 8-group
        float x1[8], x2[8];
        Vec16<__nv_bfloat16>::unpack(*reinterpret_cast<const uint4*>(kr + i0 * 2), x1);
        Vec16<__nv_bfloat16>::unpack(*reinterpret_cast<const uint4*>(kr + (i0 + HALF) * 2), x2);
        if (local) {
          const float2* c = cs + row * HALF + i0;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float2 w = c[e];
            const float a = x1[e], bb = x2[e];
            x1[e] = a * w.x - bb * w.y;
            x2[e] = bb * w.x + a * w.y;
          }
        }
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float4 q1a = *reinterpret_cast<const float4*>(&qs[h][i0]);
          const float4 q1b = *reinterpret_cast<const float4*>(&qs[h][i0 + 4]);
          const float4 q2a = *reinterpret_cast<const float4*>(&qs[h][i0 + HALF]);
          const float4 q2b = *reinterpret_cast<const float4*>(&qs[h][i0 + HALF + 4]);
          float s = acc[h];
          s = fmaf(q1a.x, x1[0], s); s = fmaf(q1a.y, x1[1], s);
          s = fmaf(q1a.z, x1[2], s); s = fmaf(q1a.w, x1[3], s);
          s = fmaf(q1b.x, x1[4], s); s = fmaf(q1b.y, x1[5], s);
          s = fmaf(q1b.z, x1[6], s); s = fmaf(q1b.w, x1[7], s);
          s = fmaf(q2a.x, x2[0], s); s = fmaf(q2a.y, x2[1], s);
          s = fmaf(q2a.z, x2[2], s); s = fmaf(q2a.w, x2[3], s);
          s = fmaf(q2b.x, x2[4], s); s = fmaf(q2b.y, x2[5], s);
          s = fmaf(q2b.z, x2[6], s); s = fmaf(q2b.w, x2[7], s);
          acc[h] = s;
        }
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float s = acc[h] + __shfl_xor_sync(0xffffffffu, acc[h], 1);
        if (hp == 0) sc[h][row] = key0 + row < k_hi ? s : -INFINITY;
      }
    }
    __syncthreads();

    // softmax and P V: warp w handles heads w, w+4, ...
#pragma unroll
    for (int a = 0; a < HPW; ++a) {
      const int h = warp + 4 * a;
      if (h >= G) break;
      const float s0 = sc[h][lane], s1 = sc[h][lane + 32];
      float mt = fmaxf(s0, s1);
#pragma unroll
      for (int off = 16; off; off >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
      const float m_new = fmaxf(m_run[a], mt);
      if (m_new == -INFINITY) continue;  // warp-uniform: nothing visible yet
      const float alpha = ex2f(m_run[a] - m_new);
      const float p0 = ex2f(s0 - m_new), p1 = ex2f(s1 - m_new);
      float ps = p0 + p1;
#pragma unroll
      for (int off = 16; off; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
      l_run[a] = l_run[a] * alpha + ps;
      m_run[a] = m_new;
      __syncwarp();
      sc[h][lane] = p0;
      sc[h][lane + 32] = p1;
      __syncwarp();
#pragma unroll
      for (int x = 0; x < VPL; ++x) o[a][x] *= alpha;
      const unsigned char* vt = sV + st * kDKeys * ROW_B + lane * VPL * 2;
#pragma unroll 8
      for (int r = 0; r < kDKeys; ++r) {
        const float p = sc[h][r];
        const uint2 w = *reinterpret_cast<const uint2*>(vt + r * ROW_B);
        o[a][0] = fmaf(p, __uint_as_float(w.x << 16), o[a][0]);
        o[a][1] = fmaf(p, __uint_as_float(w.x & 0xffff0000u), o[a][1]);
        o[a][2] = fmaf(p, __uint_as_float(w.y << 16), o[a][2]);
        o[a][3] = fmaf(p, __uint_as_float(w.y & 0xffff0000u), o[a][3]);
      }
    }
    __syncthreads();  // the stage and sc are rewritten next
  }

#pragma unroll
  for (int a = 0; a < HPW; ++a) {
    const int h = warp + 4 * a;
    if (h >= G) break;
    const int hq = g * G + h;
    const int64_t row_id = (int64_t)b * Hq + hq;  // T == 1
    if (n_split == 1) {
      const float inv = l_run[a] > 0.f ? 1.f / l_run[a] : 0.f;
      float f[4];
#pragma unroll
      for (int x = 0; x < 4; ++x) f[x] = o[a][x] * inv;
      __nv_bfloat162 lo = __floats2bfloat162_rn(f[0], f[1]), hi = __floats2bfloat162_rn(f[2], f[3]);
      uint2 pk;
      pk.x = *reinterpret_cast<uint32_t*>(&lo);
      pk.y = *reinterpret_cast<uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(out + row_id * D + lane * VPL) = pk;
    } else {
      float* po = part_o + (row_id * n_split + split) * D + lane * VPL;
      *reinterpret_cast<float4*>(po) = make_float4(o[a][0], o[a][1], o[a][2], o[a][3]);
      if (lane == 0) part_ml[row_id * n_split + split] = make_float2(m_run[a], l_run[a]);
    }
  }
}

struct DecPlan {
  int n_split;
  size_t po_bytes, ml_bytes, total;
};

DecPlan dec_plan(int B, int Hq, int H, int D, int T_loc, int m_cap) {
  DecPlan p{};
  const int64_t base = (int64_t)B * H;
  const int64_t keys = (int64_t)m_cap + T_loc;
  int64_t ns = (4LL * num_sms() + base - 1) / base;  // two resident CTAs per SM, twice over
  ns = std::min<int64_t>(ns, std::max<int64_t>(1, keys / 256));
  ns = std::min<int64_t>(ns, 64);
  p.n_split = (int)std::max<int64_t>(ns, 1);
  const size_t rows = (size_t)B * Hq;
  p.po_bytes = p.n_split > 1 ? round_up(rows * p.n_split * D * sizeof(float), 256) : 0;
  p.ml_bytes = p.n_split > 1 ? round_up(rows * p.n_split * sizeof(float2), 256) : 0;
  p.total = p.po_bytes + p.ml_bytes;
  return p;
}

template <int D, int G>
int launch_dec(int B, int T_loc, int Hq, int H, const void* q, const void* k_mem,
               const void* v_mem, const int32_t* mem_len, int m_cap, const void* k_loc,
               const void* v_loc, int pos0, float rope_base, float qscale, void* out, void* ws,
               cudaStream_t s) {
  const DecPlan p = dec_plan(B, Hq, H, D, T_loc, m_cap);
  unsigned char* w = static_cast<unsigned char*>(ws);
  float* part_o = reinterpret_cast<float*>(w);
  float2* part_ml = reinterpret_cast<float2*>(w + p.po_bytes);
  const size_t smem = (size_t)2 * kDStages * kDKeys * D * 2 + (size_t)kDKeys * (D / 2) * 8;
  auto kern = attn_decode_kernel<D, G>;
  int rc = ensure_smem_attr(reinterpret_cast<const void*>(kern), (int)smem);
  if (rc) return rc;
  const dim3 grid((unsigned)p.n_split, (unsigned)(B * H));
  kern<<<grid, kDThreads, smem, s>>>(
      T_loc, Hq, H, static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k_mem),
      static_cast<const __nv_bfloat16*>(v_mem), mem_len, m_cap,
      static_cast<const __nv_bfloat16*>(k_loc), static_cast<const __nv_bfloat16*>(v_loc), pos0,
      (double)rope_base, qscale, p.n_split, static_cast<__nv_bfloat16*>(out), part_o, part_ml);
  rc = check_launch();
  if (rc || p.n_split == 1) return rc;
  return attn_combine_bf16(B, 1, Hq, D, p.n_split, part_o, part_ml, out, s);
}

}  // namespace

bool attn_decode_supported(int T, int Hq, int H, int D) {
  if (T != 1 || D != 128 || H <= 0 || Hq % H) return false;
  const int G = Hq / H;
  return G == 1 || G == 2 || G == 4 || G == 8 || G == 16;
}

size_t attn_decode_workspace_size(int B, int T_loc, int Hq, int H, int D, int m_cap) {
  return dec_plan(B, Hq, H, D, T_loc, m_cap).total;
}

int attn_decode_launch(int B, int T_loc, int Hq, int H, int D, const void* q, const void* k_mem,
                       const void* v_mem, const int32_t* mem_len, int m_cap, const void* k_loc,
                       const void* v_loc, int pos0, float rope_base, float qscale, void* out,
                       void* ws, cudaStream_t s) {
  if (!aligned16(k_loc) || !aligned16(v_loc) || (m_cap > 0 && (!aligned16(k_mem) || !aligned16(v_mem))))
    return MSA_ERR_INVALID_ARG;
  const int G = Hq / H;
#define MSA_DEC_CASE(DD, GG)                                                                    \
  if (D == DD && G == GG)                                                                       \
    return launch_dec<DD, GG>(B, T_loc, Hq, H, q, k_mem, v_mem, mem_len, m_cap, k_loc, v_loc, \
                              pos0, rope_base, qscale, out, ws, s);
  MSA_DEC_CASE(128, 1) MSA_DEC_CASE(128, 2) MSA_DEC_CASE(128, 4) MSA_DEC_CASE(128, 8)
  MSA_DEC_CASE(128, 16)
#undef MSA_DEC_CASE
  return MSA_ERR_UNSUPPORTED;
}

}  // namespace msa
