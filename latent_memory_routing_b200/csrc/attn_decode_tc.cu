// bf16 decode attention (one query token) on the tcgen05 tensor cores, over
// [gathered memory ; local context], GQA, global RoPE offset by k.
//
// Method: "EverMind-AI/MSA: routing top-k compressed documents inside
// attention ..." (hysenlabs.com), §"Routing happens inside attention ..."
// (the selected documents' compressed K/V are concatenated with the query's
// local K/V for autoregressive decoding) and §"Document-wise RoPE resets
// every document to position zero" (global RoPE, query start offset by k).
// The query is the last of the T_loc local tokens and sees every key.
//
// Design.  Decode is HBM-bound (every K/V byte is read once); the tensor
// cores take the two contractions off the CUDA cores so that the few
// instructions left per key hide under the stream.  One CTA of 14 warps per
// (key split, batch element, KV head) serves the G query heads of the KV
// head, padded to N = 16 MMA columns:
//   * warp 0 TMA-loads 128-key K and V tiles (128B-swizzled, 64-dim blocks)
//     into a 3-stage ring -- memory tiles first, then local tiles, so no
//     tile mixes the two;
//   * warps 2, 3, 8..13 (rotators) apply RoPE to local K tiles in shared
//     memory in the relative form <R(p_q) q, R(p_k) k> = <R(Delta) q,
//     R(delta) k>: a key's rotation by its offset delta in the tile uses a
//     per-call (delta, frequency) table, and the query, rotated once per
//     tile by the tile's distance Delta to it (one complex step per tile from
//     an exact anchor), is written as the MMA's B operand; memory keys are not
//     rotated and meet R(p_q) q.  In a memory tile that ends early they zero
//     the V rows past mem_len;
//   * warp 1 issues S^T = K Q^T (M = 128 keys, N = 16, K = 128) into one of
//     two TMEM buffers and O^T += V^T P^T (M = 128 dims, N = 16, K = 128
//     keys; V read MN-major) into the O^T TMEM columns, in the order
//     S(0) S(1) | PV(0) S(2) | PV(1) S(3) ..., so the softmax of a tile runs
//     under the next tile's S;
//   * warps 4..7 (softmax, one thread per TMEM lane: a key row of S^T, a dim
//     row of O^T) turn S into P (base-2 exponent domain, the scale folded
//     into Q) against a per-head reference maximum that moves only when a
//     score exceeds it by more than 2^8 -- then O^T is rescaled in TMEM --,
//     keep per-thread partial row sums (reduced once at the end), and write
//     P^T (bf16) as the B operand of P V.
// Splits write (max, sum, O) partials that the split-KV combine kernel
// merges; a single split writes the normalised output directly.  Every wait
// is bounded; after a timeout every role walks its loop without waiting.
#include <cudaTypedefs.h>

#include <algorithm>

#include "attn_tc.cuh"
#include "msa_common.cuh"
#include "tc_ptx.cuh"

namespace msa {
namespace {

constexpr int kTK = 128;                   // keys per tile (M of S^T)
constexpr int kNH = 16;                    // MMA columns: G <= 16 heads, padded
constexpr int kDim = 128;                  // head dim
constexpr int kTStages = 3;
constexpr int kRotWarps = 8;
constexpr int kSoftWarps = 4;
constexpr int kTThreads = 32 * (2 + kRotWarps + kSoftWarps);
constexpr int kBlk = kTK * 128;            // one 64-dim block of a K or V tile: 16 KB
constexpr int kTileBytes = 2 * kBlk;       // K or V tile: 32 KB
constexpr int kStageBytes = 2 * kTileBytes;
constexpr int kQBytes = kNH * kDim * 2;    // Q [16][128] bf16: two 2 KB blocks
constexpr int kPBytes = kNH * kTK * 2;     // P^T [16][128] bf16: two 2 KB blocks
constexpr int kSmBar = 1;                  // named barrier of the softmax warps
constexpr float kRescaleLog2 = 8.f;
constexpr uint32_t kIdescS = tc::idesc_bf16_f32(kTK, kNH);
constexpr uint32_t kIdescO = tc::idesc_bf16_f32(kDim, kNH) | (1u << 15);  // A MN-major
constexpr uint32_t kTmemCols = 64;         // S buffers: 0..31, O^T: 32..47

struct DTS {  // dynamic shared memory, offsets from a 1024-byte aligned base
  static constexpr size_t RING = 0;
  static constexpr size_t QMEM = RING + (size_t)kTStages * kStageBytes;
  static constexpr size_t QT = QMEM + kQBytes;       // [2]
  static constexpr size_t P = QT + 2 * kQBytes;      // [2]
  static constexpr size_t QRAW = P + 2 * kPBytes;    // [16][128] f32, scaled raw query
  static constexpr size_t RED = QRAW + (size_t)kNH * kDim * 4;  // [4][16] f32
  static constexpr size_t FLAGS = RED + 4 * kNH * 4;            // [2][4] int
  static constexpr size_t ALLOC = FLAGS + 2 * 4 * 4 + 1024;
  static_assert(QMEM % 1024 == 0 && QT % 1024 == 0 && P % 1024 == 0, "swizzle atoms");
};

struct DTAux {
  uint64_t full[kTStages], kready[kTStages], sfree[kTStages], sfull[2], pfull[2], pvdone, odone;
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ void soft_bar() {
  asm volatile("bar.sync %0, %1;" ::"n"(kSmBar), "n"(32 * kSoftWarps) : "memory");
}
__device__ __forceinline__ float ex2a(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
// Byte offset of element (row, k) in a K-major 128B-swizzled operand of
// `rows` rows and 128 K elements (two 64-element blocks of rows x 128 B).
__device__ __forceinline__ uint32_t sw128_off(int row, int k, int rows) {
  const int kk = k & 63;
  return (uint32_t)((k >> 6) * rows * 128 + row * 128 + ((((kk >> 3) ^ (row & 7))) << 4) +
                    (kk & 7) * 2);
}

template <int G>
__global__ void __launch_bounds__(kTThreads, 1)
attn_decode_tc_kernel(const __grid_constant__ CUtensorMap tm_km,
                      const __grid_constant__ CUtensorMap tm_vm,
                      const __grid_constant__ CUtensorMap tm_kl,
                      const __grid_constant__ CUtensorMap tm_vl, int T_loc, int Hq, int H,
                      const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ mem_len,
                      int m_cap, int64_t pos0, double base, float qscale, int n_split,
                      const float2* __restrict__ cs_tab, __nv_bfloat16* __restrict__ out,
                      float* __restrict__ part_o, float2* __restrict__ part_ml,
                      int* __restrict__ status) {
  static_assert(G >= 1 && G <= kNH, "heads per KV head");
  constexpr int HALF = kDim / 2;
  extern __shared__ __align__(1024) unsigned char dsm[];
  __shared__ DTAux aux;
  unsigned char* sm = tc::smem_align<1024>(dsm);
  unsigned char* ring = sm + DTS::RING;
  unsigned char* qmem = sm + DTS::QMEM;
  unsigned char* qt = sm + DTS::QT;
  unsigned char* pbuf = sm + DTS::P;
  float* qraw = reinterpret_cast<float*>(sm + DTS::QRAW);
  float* red = reinterpret_cast<float*>(sm + DTS::RED);
  int* flags = reinterpret_cast<int*>(sm + DTS::FLAGS);

  const int split = blockIdx.x;
  const int b = blockIdx.y / H, g = blockIdx.y % H;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int M = min(max(mem_len[b], 0), m_cap);
  const int n_mt = (M + kTK - 1) / kTK;
  const int n_all = n_mt + (T_loc + kTK - 1) / kTK;
  const int j_lo = (int)((int64_t)split * n_all / n_split);
  const int j_hi = (int)((int64_t)(split + 1) * n_all / n_split);
  const int nt = j_hi - j_lo;
  if (nt <= 0) {  // an empty split: neutral partial
    for (int e = tid; e < G * kDim; e += kTThreads) {
      const int64_t row_id = (int64_t)b * Hq + g * G + e / kDim;
      part_o[(row_id * n_split + split) * kDim + e % kDim] = 0.f;
      if (e % kDim == 0) part_ml[row_id * n_split + split] = make_float2(-INFINITY, 0.f);
    }
    return;
  }
  auto tile_mem = [&](int jj) { return jj < n_mt; };
  auto tile_key0 = [&](int jj) { return jj < n_mt ? jj * kTK : (jj - n_mt) * kTK; };
  auto tile_valid = [&](int jj) {
    return jj < n_mt ? min(kTK, M - jj * kTK) : min(kTK, T_loc - (jj - n_mt) * kTK);
  };

  if (tid == 0) {
    for (int i = 0; i < kTStages; ++i) {
      tc::mbar_init(&aux.full[i], 1);
      tc::mbar_init(&aux.kready[i], kRotWarps);
      tc::mbar_init(&aux.sfree[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&aux.sfull[i], 1);
      tc::mbar_init(&aux.pfull[i], kSoftWarps);
    }
    tc::mbar_init(&aux.pvdone, 1);
    tc::mbar_init(&aux.odone, 1);
    aux.abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(&aux.tmem_base, kTmemCols);
    tc::tmem_relinquish();
  }
  // zero the per-tile query buffers and P^T (rows >= G stay zero), keep the
  // scaled raw query, and build R(p_q) q for the memory tiles (all 16 rows)
  for (int e = tid; e < (2 * kQBytes + 2 * kPBytes) / 16; e += kTThreads)
    reinterpret_cast<uint4*>(qt)[e] = make_uint4(0, 0, 0, 0);
  for (int e = tid; e < G * kDim; e += kTThreads)
    qraw[e] = __bfloat162float(q[((int64_t)b * Hq + g * G) * kDim + e]) * qscale;
  if (n_mt > j_lo) {
    for (int e = tid; e < kNH * HALF; e += kTThreads) {
      const int h = e / HALF, i = e % HALF;
      float y1 = 0.f, y2 = 0.f;
      if (h < G) {
        const __nv_bfloat16* qp = q + ((int64_t)b * Hq + g * G + h) * kDim;
        const float x1 = __bfloat162float(qp[i]) * qscale;
        const float x2 = __bfloat162float(qp[i + HALF]) * qscale;
        const float2 c = rope_cs(pos0 + T_loc - 1, rope_inv_freq(base, i, kDim));
        y1 = x1 * c.x - x2 * c.y;
        y2 = x2 * c.x + x1 * c.y;
      }
      *reinterpret_cast<__nv_bfloat16*>(qmem + sw128_off(h, i, kNH)) = __float2bfloat16(y1);
      *reinterpret_cast<__nv_bfloat16*>(qmem + sw128_off(h, i + HALF, kNH)) =
          __float2bfloat16(y2);
    }
  }
  tc::fence_proxy_async_smem();
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = aux.tmem_base;
  volatile int* abort_flag = &aux.abort_flag;
  auto wait_or_abort = [&](uint64_t* bar, uint32_t parity) {
    if (*abort_flag) return;
    if (!tc::mbar_wait(bar, parity)) {
      record_error(status, MSA_ERR_TIMEOUT);
      *abort_flag = 1;
    }
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int issued = 0;
      for (int j = 0; j < nt; ++j) {
        const int st = j % kTStages;
        wait_or_abort(&aux.sfree[st], ((j / kTStages) & 1) ^ 1);
        if (*abort_flag) break;
        const int jj = j_lo + j;
        unsigned char* kd = ring + (size_t)st * kStageBytes;
        const bool mem = tile_mem(jj);
        const int row0 = mem ? b * m_cap + tile_key0(jj) : b * T_loc + tile_key0(jj);
        const CUtensorMap* mk = mem ? &tm_km : &tm_kl;
        const CUtensorMap* mv = mem ? &tm_vm : &tm_vl;
        tc::mbar_arrive_expect_tx(&aux.full[st], kStageBytes);
        tc::tma_load_3d(kd, mk, &aux.full[st], 0, g, row0);
        tc::tma_load_3d(kd + kBlk, mk, &aux.full[st], 64, g, row0);
        tc::tma_load_3d(kd + kTileBytes, mv, &aux.full[st], 0, g, row0);
        tc::tma_load_3d(kd + kTileBytes + kBlk, mv, &aux.full[st], 64, g, row0);
        ++issued;
      }
      for (int v = issued > kTStages ? issued - kTStages : 0; v < issued; ++v)
        tc::mbar_wait(&aux.full[v % kTStages], (v / kTStages) & 1);
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      auto issue_s = [&](int j) {
        const int st = j % kTStages;
        wait_or_abort(&aux.kready[st], (j / kTStages) & 1);
        tc::tc_fence_after();
        const uint32_t a0 = tc::smem_u32(ring + (size_t)st * kStageBytes);
        const uint32_t b0 = tc::smem_u32(tile_mem(j_lo + j) ? qmem : qt + (j & 1) * kQBytes);
#pragma unroll
        for (int kk = 0; kk < kDim / 16; ++kk) {
          const uint32_t koff = (kk & 3) * 32;
          tc::mma_bf16_ss(tmem + (j & 1) * kNH,
                          tc::sdesc_kmajor_sw128(a0 + (kk >> 2) * kBlk + koff),
                          tc::sdesc_kmajor_sw128(b0 + (kk >> 2) * (kNH * 128) + koff), kIdescS,
                          kk > 0 ? 1u : 0u);
        }
        tc::mma_commit(&aux.sfull[j & 1]);
      };
      auto issue_pv = [&](int j) {
        const int st = j % kTStages;
        wait_or_abort(&aux.pfull[j & 1], (j >> 1) & 1);
        tc::tc_fence_after();
        const uint32_t v0 = tc::smem_u32(ring + (size_t)st * kStageBytes + kTileBytes);
        const uint32_t p0 = tc::smem_u32(pbuf + (j & 1) * kPBytes);
#pragma unroll
        for (int kk = 0; kk < kTK / 16; ++kk)
          tc::mma_bf16_ss(tmem + 2 * kNH, tc::sdesc_mnmajor_sw128(v0 + kk * 16 * 128, kBlk),
                          tc::sdesc_kmajor_sw128(p0 + (kk >> 2) * (kNH * 128) + (kk & 3) * 32),
                          kIdescO, (j > 0 || kk > 0) ? 1u : 0u);
        tc::mma_commit(&aux.sfree[st]);
        tc::mma_commit(&aux.pvdone);
        if (j == nt - 1) tc::mma_commit(&aux.odone);
      };
      issue_s(0);
      if (nt > 1) issue_s(1);
      for (int j = 0; j < nt; ++j) {
        issue_pv(j);
        if (j + 2 < nt) issue_s(j + 2);
      }
    }
  } else if (warp >= 4 && warp < 4 + kSoftWarps) {
    // ------------------------------------------------------------- softmax
    const int w4 = warp - 4;            // TMEM lane quarter
    const int r = w4 * 32 + lane;       // key row of S^T, dim row of O^T
    const uint32_t lane_addr = (uint32_t)(w4 * 32) << 16;
    float m_ref[G], l_part[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      m_ref[h] = -INFINITY;
      l_part[h] = 0.f;
    }
    for (int j = 0; j < nt; ++j) {
      wait_or_abort(&aux.sfull[j & 1], (j >> 1) & 1);
      tc::tc_fence_after();
      const int jj = j_lo + j;
      const bool valid = r < tile_valid(jj);
      uint32_t sv[16];
      tc::tmem_ld16(tmem + lane_addr + (j & 1) * kNH, sv);
      tc::tmem_ld_wait();
      float s[G];
      bool need = false;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        s[h] = valid ? __uint_as_float(sv[h]) : -INFINITY;
        need |= s[h] > m_ref[h] + kRescaleLog2;
      }
      const int any_w = __any_sync(0xffffffffu, need);
      if (lane == 0) flags[(j & 1) * 4 + w4] = any_w;
      soft_bar();
      const bool any = flags[(j & 1) * 4] | flags[(j & 1) * 4 + 1] | flags[(j & 1) * 4 + 2] |
                       flags[(j & 1) * 4 + 3];
      if (any) {  // uniform: new reference maxima from the tile's maxima
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float mx = s[h];
#pragma unroll
          for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
          if (lane == 0) red[w4 * kNH + h] = mx;
        }
        soft_bar();
        float alpha[G];
        bool rescale = false;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float mt = fmaxf(fmaxf(red[h], red[kNH + h]), fmaxf(red[2 * kNH + h], red[3 * kNH + h]));
          alpha[h] = 1.f;
          if (mt > m_ref[h] + kRescaleLog2) {
            alpha[h] = m_ref[h] == -INFINITY ? 0.f : ex2a(m_ref[h] - mt);
            m_ref[h] = mt;
            rescale = true;
          }
          l_part[h] *= alpha[h];
        }
        if (rescale && j > 0) {
          // O^T holds P V of tiles < j: wait for the last of them, then
          // scale each head's column (the TMEM columns of this thread's dim)
          wait_or_abort(&aux.pvdone, (j - 1) & 1);
          tc::tc_fence_after();
          uint32_t ov[16];
          tc::tmem_ld16(tmem + lane_addr + 2 * kNH, ov);
          tc::tmem_ld_wait();
#pragma unroll
          for (int h = 0; h < G; ++h) ov[h] = __float_as_uint(__uint_as_float(ov[h]) * alpha[h]);
          tmem_st16(tmem + lane_addr + 2 * kNH, ov);
          tmem_st_wait();
        }
      }
      // P^T column of this key (buffer j&1: its previous reader, P V of tile
      // j-2, completed before S(j) was issued)
      unsigned char* pb = pbuf + (j & 1) * kPBytes;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float p = (valid && m_ref[h] != -INFINITY) ? ex2a(s[h] - m_ref[h]) : 0.f;
        l_part[h] += p;
        *reinterpret_cast<__nv_bfloat16*>(pb + sw128_off(h, r, kNH)) = __float2bfloat16(p);
      }
      tc::fence_proxy_async_smem();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&aux.pfull[j & 1]);
    }
    wait_or_abort(&aux.odone, 0);
    tc::tc_fence_after();
    // row sums: per-thread partials reduced over the 128 key lanes
    soft_bar();  // every thread is past its last read of red
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float v = l_part[h];
#pragma unroll
      for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) red[w4 * kNH + h] = v;
    }
    soft_bar();
    uint32_t ov[16];
    tc::tmem_ld16(tmem + lane_addr + 2 * kNH, ov);
    tc::tmem_ld_wait();
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float l = red[h] + red[kNH + h] + red[2 * kNH + h] + red[3 * kNH + h];
      const int64_t row_id = (int64_t)b * Hq + g * G + h;  // T == 1
      const float o = __uint_as_float(ov[h]);
      if (n_split == 1) {
        out[row_id * kDim + r] = __float2bfloat16(l > 0.f ? o / l : 0.f);
      } else {
        part_o[(row_id * n_split + split) * kDim + r] = o;
        if (r == 0) part_ml[row_id * n_split + split] = make_float2(m_ref[h], l);
      }
    }
  } else {
    // ------------------------------------------------------------ rotators
    const int rt = (warp < 4 ? warp - 2 : warp - 6) * 32 + lane;  // 0 .. 255
    const int c = rt & 7, r0 = rt >> 3;  // 16-byte chunk, first of four rows
    float2 cs[4][8];                     // (cos, sin) of delta = r0 + 32 q, pair 8c + e
#pragma unroll
    for (int qq = 0; qq < 4; ++qq)
#pragma unroll
      for (int e = 0; e < 8; ++e) cs[qq][e] = cs_tab[(r0 + 32 * qq) * HALF + 8 * c + e];
    const int i_q = rt % HALF;  // query pair this thread rotates
    const double wq = rope_inv_freq(base, i_q, kDim);
    const float2 qstep = rope_cs(kTK, wq);
    float2 qcs = make_float2(1.f, 0.f);
    bool anchored = false;
    for (int j = 0; j < nt; ++j) {
      const int st = j % kTStages, jj = j_lo + j;
      wait_or_abort(&aux.full[st], (j / kTStages) & 1);
      unsigned char* kt = ring + (size_t)st * kStageBytes;
      const int n_valid = tile_valid(jj);
      if (!tile_mem(jj)) {
        // the query for this tile: R(Delta) q into buffer j&1, whose last
        // reader S(j-2) must be done
        if (j >= 2) wait_or_abort(&aux.sfull[j & 1], ((j - 2) >> 1) & 1);
        const int Delta = T_loc - 1 - tile_key0(jj);
        if (!anchored) {
          qcs = rope_cs(Delta, wq);
          anchored = true;
        } else {  // Delta fell by kTK: multiply by e^{-i kTK w}
          const float cc = qcs.x * qstep.x + qcs.y * qstep.y;
          qcs.y = qcs.y * qstep.x - qcs.x * qstep.y;
          qcs.x = cc;
        }
        unsigned char* qb = qt + (j & 1) * kQBytes;
        for (int e = rt; e < G * HALF; e += 32 * kRotWarps) {
          const int h = e / HALF;
          const float x1 = qraw[h * kDim + i_q], x2 = qraw[h * kDim + i_q + HALF];
          *reinterpret_cast<__nv_bfloat16*>(qb + sw128_off(h, i_q, kNH)) =
              __float2bfloat16(x1 * qcs.x - x2 * qcs.y);
          *reinterpret_cast<__nv_bfloat16*>(qb + sw128_off(h, i_q + HALF, kNH)) =
              __float2bfloat16(x2 * qcs.x + x1 * qcs.y);
        }
        // R(delta) k for this thread's four rows, 8 pairs each: dims
        // 8c..8c+7 (first block) and their partners 64 + 8c.. (second block,
        // same swizzled offset)
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
          const int rr = r0 + 32 * qq;
          const uint32_t off = rr * 128 + ((c ^ (rr & 7)) << 4);
          uint4* p1 = reinterpret_cast<uint4*>(kt + off);
          uint4* p2 = reinterpret_cast<uint4*>(kt + kBlk + off);
          float x1[8], x2[8], y1[8], y2[8];
          Vec16<__nv_bfloat16>::unpack(*p1, x1);
          Vec16<__nv_bfloat16>::unpack(*p2, x2);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            y1[e] = x1[e] * cs[qq][e].x - x2[e] * cs[qq][e].y;
            y2[e] = x2[e] * cs[qq][e].x + x1[e] * cs[qq][e].y;
          }
          *p1 = Vec16<__nv_bfloat16>::pack(y1);
          *p2 = Vec16<__nv_bfloat16>::pack(y2);
        }
      } else if (n_valid < kTK) {
        // memory rows past mem_len hold whatever the caller's buffer holds:
        // zero their V so that 0 * V stays 0 in P V
        unsigned char* vt = kt + kTileBytes;
        for (int e = rt; e < (kTK - n_valid) * 16; e += 32 * kRotWarps) {
          const int rr = n_valid + e / 16, cc = e % 16;
          *reinterpret_cast<uint4*>(vt + (cc >> 3) * kBlk + rr * 128 + ((cc & 7) << 4)) =
              make_uint4(0, 0, 0, 0);
        }
      }
      tc::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&aux.kready[st]);
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

// (cos, sin) of delta * w_i for delta in [0, 128), i in [0, 64): exact
// angles (reduced in double), once per call.
__global__ void decode_cs_table_kernel(double base, float2* __restrict__ tab) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e < kTK * (kDim / 2)) tab[e] = rope_cs(e / (kDim / 2), rope_inv_freq(base, e % (kDim / 2), kDim));
}

struct DTPlan {
  int n_split;
  size_t tab_bytes, po_bytes, ml_bytes, total;
};

// Key splits: the grid runs in waves of one CTA per SM and a CTA pays a
// pipeline start; take the split count with the fewest tile-slots per SM
// (waves x tiles per CTA), plus half a tile per CTA for the start.
DTPlan dt_plan(int B, int Hq, int H, int T_loc, int m_cap) {
  DTPlan p{};
  const int64_t base = (int64_t)B * H;
  const int64_t tiles = ((int64_t)m_cap + kTK - 1) / kTK + (T_loc + kTK - 1) / kTK;
  const int64_t sms = std::max(1, num_sms());
  double best = 1e30;
  int pick = 1;
  for (int ns = 1; ns <= std::min<int64_t>(tiles, 32); ++ns) {
    const int64_t waves = (base * ns + sms - 1) / sms;
    const double cost = (double)waves * ((tiles + ns - 1) / ns + 0.5);
    if (cost < best - 1e-9) {
      best = cost;
      pick = ns;
    }
  }
  p.n_split = pick;
  p.tab_bytes = round_up((size_t)kTK * (kDim / 2) * sizeof(float2), 256);
  const size_t rows = (size_t)B * Hq;
  p.po_bytes = p.n_split > 1 ? round_up(rows * p.n_split * kDim * sizeof(float), 256) : 0;
  p.ml_bytes = p.n_split > 1 ? round_up(rows * p.n_split * sizeof(float2), 256) : 0;
  p.total = p.tab_bytes + p.po_bytes + p.ml_bytes;
  return p;
}

template <int G>
int launch_dtc(int B, int T_loc, int Hq, int H, const void* q, const void* k_mem,
               const void* v_mem, const int32_t* mem_len, int m_cap, const void* k_loc,
               const void* v_loc, int pos0, float rope_base, float qscale, void* out, void* ws,
               cudaStream_t s) {
  const DTPlan p = dt_plan(B, Hq, H, T_loc, m_cap);
  unsigned char* w = static_cast<unsigned char*>(ws);
  float2* tab = reinterpret_cast<float2*>(w);
  float* part_o = reinterpret_cast<float*>(w + p.tab_bytes);
  float2* part_ml = reinterpret_cast<float2*>(w + p.tab_bytes + p.po_bytes);
  decode_cs_table_kernel<<<(kTK * (kDim / 2) + 255) / 256, 256, 0, s>>>((double)rope_base, tab);
  int rc = check_launch();
  if (rc) return rc;
  CUtensorMap tkm, tvm, tkl, tvl;
  const bool has_mem = m_cap > 0;
  const int64_t mem_rows = has_mem ? (int64_t)B * m_cap : (int64_t)B * T_loc;
  if (!tma_map_sw128_bf16(&tkm, has_mem ? k_mem : k_loc, kDim, H, mem_rows, 1, kTK) ||
      !tma_map_sw128_bf16(&tvm, has_mem ? v_mem : v_loc, kDim, H, mem_rows, 1, kTK) ||
      !tma_map_sw128_bf16(&tkl, k_loc, kDim, H, (int64_t)B * T_loc, 1, kTK) ||
      !tma_map_sw128_bf16(&tvl, v_loc, kDim, H, (int64_t)B * T_loc, 1, kTK))
    return note_cuda(cudaErrorInvalidValue);
  auto kern = attn_decode_tc_kernel<G>;
  rc = ensure_smem_attr(reinterpret_cast<const void*>(kern), (int)DTS::ALLOC);
  if (rc) return rc;
  const dim3 grid((unsigned)p.n_split, (unsigned)(B * H));
  kern<<<grid, kTThreads, DTS::ALLOC, s>>>(tkm, tvm, tkl, tvl, T_loc, Hq, H,
                                           static_cast<const __nv_bfloat16*>(q), mem_len, m_cap,
                                           pos0, (double)rope_base, qscale, p.n_split, tab,
                                           static_cast<__nv_bfloat16*>(out), part_o, part_ml,
                                           device_status_ptr());
  rc = check_launch();
  if (rc || p.n_split == 1) return rc;
  return attn_combine_bf16(B, 1, Hq, kDim, p.n_split, part_o, part_ml, out, s);
}

}  // namespace

bool attn_decode_tc_supported(int T, int Hq, int H, int D) {
  if (T != 1 || D != kDim || H <= 0 || Hq % H) return false;
  const int G = Hq / H;
  return G == 1 || G == 2 || G == 4 || G == 8 || G == 16;
}

size_t attn_decode_tc_workspace_size(int B, int T_loc, int Hq, int H, int D, int m_cap) {
  (void)D;
  return dt_plan(B, Hq, H, T_loc, m_cap).total;
}

int attn_decode_tc_launch(int B, int T_loc, int Hq, int H, int D, const void* q,
                          const void* k_mem, const void* v_mem, const int32_t* mem_len,
                          int m_cap, const void* k_loc, const void* v_loc, int pos0,
                          float rope_base, float qscale, void* out, void* ws, cudaStream_t s) {
  if (!aligned16(k_loc) || !aligned16(v_loc) ||
      (m_cap > 0 && (!aligned16(k_mem) || !aligned16(v_mem))))
    return MSA_ERR_INVALID_ARG;
  if ((int64_t)B * H > 65535 || (int64_t)B * std::max(m_cap, T_loc) > INT32_MAX)
    return MSA_ERR_UNSUPPORTED;
  const int G = Hq / H;
#define MSA_DTC_CASE(GG)                                                                    \
  if (D == kDim && G == GG)                                                                 \
    return launch_dtc<GG>(B, T_loc, Hq, H, q, k_mem, v_mem, mem_len, m_cap, k_loc, v_loc, \
                          pos0, rope_base, qscale, out, ws, s);
  MSA_DTC_CASE(1) MSA_DTC_CASE(2) MSA_DTC_CASE(4) MSA_DTC_CASE(8) MSA_DTC_CASE(16)
#undef MSA_DTC_CASE
  return MSA_ERR_UNSUPPORTED;
}

}  // namespace msa
