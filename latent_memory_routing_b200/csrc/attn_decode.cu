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
// share the KV head; about 40 KB of shared memory, so four CTAs per SM:
//   * 32-key tiles of K and V stream with 16-byte cp.async through a 3-stage
//     shared ring;
//   * four threads per key row, each owning 16 of the 64 rotate-half pairs.
//     A local row is rotated in registers with the (cos, sin) of its
//     position, also in registers: computed exactly (angle reduced in double)
//     at the CTA's first tile holding a local row, then advanced by one
//     complex multiply per tile (the row moves 32 positions), so the drift
//     over a split stays at a few 1e-7.  The rotated quarter-row is dotted
//     with the G rotated queries (shared memory) and the four partial dots
//     are summed with two shuffles;
//   * one warp per query head runs the online softmax over the tile's 32
//     scores (one per lane) and accumulates O, 4 dims per lane, from the V
//     tile with packed fp32 FMAs;
//   * splits write (max, sum, O) partials that the split-KV combine kernel
//     merges; a single split writes the normalised output directly.
#include <algorithm>

#include "attn_tc.cuh"
#include "msa_common.cuh"

namespace msa {
namespace {

constexpr int kDThreads = 128;
constexpr int kDKeys = 32;   // keys per tile
constexpr int kDStages = 3;

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

// o += p * (lo, hi) on a packed fp32 pair.
__device__ __forceinline__ void fma2(unsigned long long& o, unsigned long long p2,
                                     unsigned long long v2) {
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(o) : "l"(p2), "l"(v2));
}
__device__ __forceinline__ unsigned long long bf2_to_f2(uint32_t w) {
  return ((unsigned long long)(w & 0xffff0000u) << 32) | (unsigned long long)(w << 16);
}

template <int D, int G>
__global__ void __launch_bounds__(kDThreads, 4)
attn_decode_kernel(int T_loc, int Hq, int H, const __nv_bfloat16* __restrict__ q,
                   const __nv_bfloat16* __restrict__ k_mem,
                   const __nv_bfloat16* __restrict__ v_mem, const int32_t* __restrict__ mem_len,
                   int m_cap, const __nv_bfloat16* __restrict__ k_loc,
                   const __nv_bfloat16* __restrict__ v_loc, int64_t pos0, double base,
                   float qscale, int n_split, __nv_bfloat16* __restrict__ out,
                   float* __restrict__ part_o, float2* __restrict__ part_ml) {
  static_assert(D == 128, "four output dims per lane, 16 pairs per thread");
  constexpr int HALF = D / 2;
  constexpr int QP = 16;       // pairs per thread (four threads per row)
  constexpr int ROW_B = D * 2;
  extern __shared__ __align__(16) unsigned char dsm[];
  unsigned char* sK = dsm;                                 // [stage][32 rows][D] bf16
  unsigned char* sV = dsm + kDStages * kDKeys * ROW_B;     // [stage][32 rows][D] bf16
  __shared__ __align__(16) float qs[G][D];   // rotated, scaled queries
  __shared__ float sc[G][kDKeys];            // tile scores
  __shared__ double wf[HALF];                // inverse frequencies
  __shared__ float2 stepw[HALF];             // e^{i 32 w_i}: one tile forward

  const int split = blockIdx.x;
  const int b = blockIdx.y / H, g = blockIdx.y % H;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int M = min(max(mem_len[b], 0), m_cap);
  const int n_keys = M + T_loc;
  const int per = (n_keys + n_split - 1) / n_split;
  const int k_lo = min(n_keys, split * per), k_hi = min(n_keys, k_lo + per);
  const int n_tiles = (k_hi - k_lo + kDKeys - 1) / kDKeys;

  for (int i = tid; i < HALF; i += kDThreads) {
    wf[i] = rope_inv_freq(base, i, D);
    stepw[i] = rope_cs(kDKeys, wf[i]);
  }
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

  constexpr int HPW = (G + 3) / 4;  // heads per warp in the softmax
  float m_run[HPW], l_run[HPW];
  unsigned long long o2[HPW][2];    // 4 output dims per lane, packed pairs
#pragma unroll
  for (int a = 0; a < HPW; ++a) {
    m_run[a] = -INFINITY;
    l_run[a] = 0.f;
    o2[a][0] = o2[a][1] = 0ull;
  }

  const int row = tid >> 2, qq = tid & 3;  // key row and pair quarter
  const int i0 = qq * QP;                  // first pair of this thread
  float cr[QP], sr[QP];                    // rotation of this row
  bool anchored = false;
#pragma unroll
  for (int e = 0; e < QP; ++e) {
    cr[e] = 1.f;
    sr[e] = 0.f;
  }
  __syncthreads();

#pragma unroll 1
  for (int t = 0; t < kDStages - 1; ++t)
    if (t < n_tiles) load_tile(t, t);
    else cp_async_commit();

#pragma unroll 1
  for (int t = 0; t < n_tiles; ++t) {
    const int st = t % kDStages;
    const int key0 = k_lo + t * kDKeys;
    if (t + kDStages - 1 < n_tiles) load_tile(t + kDStages - 1, (t + kDStages - 1) % kDStages);
    else cp_async_commit();
    cp_async_wait<kDStages - 1>();
    __syncthreads();

    // this row's rotation: exact at the first tile holding a local row, then
    // one complex multiply per tile
    const bool tile_local = key0 + kDKeys > M;
    if (tile_local) {
      if (!anchored) {
        const int64_t p = pos0 + (int64_t)(key0 + row - M);
#pragma unroll
        for (int e = 0; e < QP; ++e) {
          const float2 c = rope_cs(p, wf[i0 + e]);
          cr[e] = c.x;
          sr[e] = c.y;
        }
        anchored = true;
      } else {
#pragma unroll
        for (int e = 0; e < QP; ++e) {
          const float2 w = stepw[i0 + e];
          const float c = cr[e] * w.x - sr[e] * w.y;
          sr[e] = cr[e] * w.y + sr[e] * w.x;
          cr[e] = c;
        }
      }
    }

    // partial dot of this quarter-row with each query head
    {
      const unsigned char* kr = sK + (st * kDKeys + row) * ROW_B;
      float x1[QP], x2[QP];
#pragma unroll
      for (int v = 0; v < QP / 8; ++v) {
        Vec16<__nv_bfloat16>::unpack(*reinterpret_cast<const uint4*>(kr + (i0 + 8 * v) * 2),
                                     x1 + 8 * v);
        Vec16<__nv_bfloat16>::unpack(
            *reinterpret_cast<const uint4*>(kr + (i0 + 8 * v + HALF) * 2), x2 + 8 * v);
      }
      if (key0 + row >= M) {
#pragma unroll
        for (int e = 0; e < QP; ++e) {
          const float a = x1[e], bb = x2[e];
          x1[e] = a * cr[e] - bb * sr[e];
          x2[e] = bb * cr[e] + a * sr[e];
        }
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float s = 0.f;
#pragma unroll
        for (int v = 0; v < QP / 4; ++v) {
          const float4 a = *reinterpret_cast<const float4*>(&qs[h][i0 + 4 * v]);
          const float4 c = *reinterpret_cast<const float4*>(&qs[h][i0 + 4 * v + HALF]);
          s = fmaf(a.x, x1[4 * v], s);
          s = fmaf(a.y, x1[4 * v + 1], s);
          s = fmaf(a.z, x1[4 * v + 2], s);
          s = fmaf(a.w, x1[4 * v + 3], s);
          s = fmaf(c.x, x2[4 * v], s);
          s = fmaf(c.y, x2[4 * v + 1], s);
          s = fmaf(c.z, x2[4 * v + 2], s);
          s = fmaf(c.w, x2[4 * v + 3], s);
        }
        s += __shfl_xor_sync(0xffffffffu, s, 1);
        s += __shfl_xor_sync(0xffffffffu, s, 2);
        if (qq == 0) sc[h][row] = key0 + row < k_hi ? s : -INFINITY;
      }
    }
    __syncthreads();

    // softmax and P V: warp w handles heads w, w+4, ...; lane = key row
#pragma unroll
    for (int a = 0; a < HPW; ++a) {
      const int h = warp + 4 * a;
      if (h >= G) break;
      const float s = sc[h][lane];
      float mt = s;
#pragma unroll
      for (int off = 16; off; off >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
      const float m_new = fmaxf(m_run[a], mt);
      if (m_new == -INFINITY) continue;  // warp-uniform: nothing visible yet
      const float alpha = ex2f(m_run[a] - m_new);
      const float p = ex2f(s - m_new);
      float ps = p;
#pragma unroll
      for (int off = 16; off; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
      l_run[a] = l_run[a] * alpha + ps;
      m_run[a] = m_new;
      const unsigned long long al2 =
          ((unsigned long long)__float_as_uint(alpha) << 32) | __float_as_uint(alpha);
      unsigned long long z = 0ull;
      asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(z) : "l"(o2[a][0]), "l"(al2));
      o2[a][0] = z;
      asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(z) : "l"(o2[a][1]), "l"(al2));
      o2[a][1] = z;
      const unsigned char* vt = sV + st * kDKeys * ROW_B + lane * 8;
#pragma unroll 8
      for (int r = 0; r < kDKeys; ++r) {
        const float pr = __shfl_sync(0xffffffffu, p, r);
        const unsigned long long p2 =
            ((unsigned long long)__float_as_uint(pr) << 32) | __float_as_uint(pr);
        const uint2 w = *reinterpret_cast<const uint2*>(vt + r * ROW_B);
        fma2(o2[a][0], p2, bf2_to_f2(w.x));
        fma2(o2[a][1], p2, bf2_to_f2(w.y));
      }
    }
    __syncthreads();  // the stage and sc are rewritten next
  }
  cp_async_wait<0>();

#pragma unroll
  for (int a = 0; a < HPW; ++a) {
    const int h = warp + 4 * a;
    if (h >= G) break;
    const int64_t row_id = (int64_t)b * Hq + g * G + h;  // T == 1
    const float o0 = __uint_as_float((uint32_t)o2[a][0]), o1 = __uint_as_float((uint32_t)(o2[a][0] >> 32));
    const float o2v = __uint_as_float((uint32_t)o2[a][1]), o3 = __uint_as_float((uint32_t)(o2[a][1] >> 32));
    if (n_split == 1) {
      const float inv = l_run[a] > 0.f ? 1.f / l_run[a] : 0.f;
      __nv_bfloat162 lo = __floats2bfloat162_rn(o0 * inv, o1 * inv);
      __nv_bfloat162 hi = __floats2bfloat162_rn(o2v * inv, o3 * inv);
      uint2 pk;
      pk.x = *reinterpret_cast<uint32_t*>(&lo);
      pk.y = *reinterpret_cast<uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(out + row_id * D + lane * 4) = pk;
    } else {
      float* po = part_o + (row_id * n_split + split) * D + lane * 4;
      *reinterpret_cast<float4*>(po) = make_float4(o0, o1, o2v, o3);
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
  int64_t ns = (8LL * num_sms() + base - 1) / base;  // four resident CTAs per SM, twice over
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
  auto kern = attn_decode_kernel<D, G>;
  const size_t smem = (size_t)2 * kDStages * kDKeys * D * 2;
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
