// bf16 prefill attention over [gathered memory ; local causal context] on the
// sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Method: "EverMind-AI/MSA: routing top-k compressed documents inside
// attention ..." (hysenlabs.com), §"Routing happens inside attention ..."
// (the selected documents' compressed K/V are concatenated ahead of the
// query's local K/V) and §"Document-wise RoPE resets every document to
// position zero" (global RoPE whose query start is offset by k).  Memory rows
// keep their document-wise rotation; local keys are causal.
//
// Design.
//   * rope_prep_kernel rotates Q (to pos0 + T_loc - T + i) and the local K
//     (to pos0 + j) once per call into bf16 workspace copies, one launch,
//     cos/sin per position built in shared memory (angles reduced in double).
//   * attn_tc_kernel: one CTA per (128 query rows, KV head, batch, key split;
//     up to 3 splits of the key tiles, merged by the split-KV combine
//     kernel, when there are too few row tiles to fill the SMs).  GQA rows
//     are packed as (token, head of the group): a TMA box of
//     {64 d, G heads, 128/G tokens} lands as 128 rows of 128 B -- the Q tile
//     of all G query heads sharing one KV head.  Key tiles of 128 rows come
//     first from the memory (mem_len rows) then from the local context
//     (up to the block's last visible key), each as K and V TMA boxes.
//     - warp 0 (one lane): TMA producer, 2-stage K/V ring;
//     - warp 1 (one lane): tcgen05.mma S = Q K^T (M=128, N=128 keys, K=D)
//       into one of two TMEM buffers, and O += P V (M=128, N=D, K=128 keys,
//       V read MN-major straight from its TMA tile) into the TMEM output
//       accumulator; the S of tile j+1 is issued before the P V of tile j;
//     - warps 2..5 (one thread per row): online softmax in fp32 -- the
//       tile's scores read once from TMEM, masked row maximum, p = 2^(s - m)
//       (SFU ex2) written as bf16 into a double-buffered shared P tile
//       (128B-swizzled, the MMA's A operand), row sum.  O accumulates in
//       TMEM; a row rescales O and its sum only when its maximum grows by
//       more than 2^8 (then p <= 256 meanwhile), which after the first tiles
//       is rare.
//   * Every mbarrier wait is bounded; a timeout records MSA_ERR_TIMEOUT and
//     all roles finish their loops without waiting.
#include <cudaTypedefs.h>

#include <algorithm>

#include "attn_tc.cuh"
#include "msa_common.cuh"
#include "tc_ptx.cuh"

namespace msa {
namespace {

constexpr int kRows = 128;   // query rows per CTA (MMA M)
constexpr int kKeys = 128;   // keys per tile (MMA N of S, K of P V)
constexpr int kSoftWarps = 4;
constexpr int kThreads = 64 + 32 * kSoftWarps;
constexpr int kStages = 2;

template <int D>
struct ACfg {
  static constexpr int KB = D / 64;
  static constexpr int Q_BYTES = KB * kRows * 128;
  static constexpr int K_BYTES = KB * kKeys * 128;
  static constexpr int V_BYTES = KB * kKeys * 128;
  static constexpr int STAGE = K_BYTES + V_BYTES;
  static constexpr int P_BYTES = 2 * kRows * 128;  // 128 keys x bf16 = 2 K blocks
  static constexpr size_t SMEM = 1024 + Q_BYTES + kStages * STAGE + 2 * P_BYTES;
  static constexpr uint32_t TMEM_COLS = 512;
  // S: M=128, N=128 keys, A (Q) and B (K) K-major
  static constexpr uint32_t IDESC_S = tc::idesc_bf16_f32(kRows, kKeys);
  // O: M=128, N=D, A (P) K-major, B (V) MN-major (bit 16)
  static constexpr uint32_t IDESC_O = tc::idesc_bf16_f32(kRows, D) | (1u << 16);
};

struct AAux {
  uint64_t q_full, kv_full[kStages], kv_empty[kStages], s_full[2], s_empty[2], p_full[2],
      o_full;
  uint32_t tmem_base;
  int abort_flag;
};

// UMMA descriptor of an MN-major, 128B-swizzled operand whose MN extent is
// split in 64-element (128 B) column blocks `lbo` bytes apart and whose K
// rows are 128 B apart (8-row swizzle atoms 1024 B apart): the layout of a
// TMA box {64 MN, rows K} stored block after block.
__device__ __forceinline__ uint64_t sdesc_mnmajor_sw128(uint32_t smem_addr, uint32_t lbo) {
  return (uint64_t)((smem_addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// 2^x by the SFU (ex2.approx, ~2 ulp); its result feeds a bf16 P tile.
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
      "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
      "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_km,
               const __grid_constant__ CUtensorMap tm_vm, const __grid_constant__ CUtensorMap tm_kl,
               const __grid_constant__ CUtensorMap tm_vl, int T, int T_loc, int Hq, int H, int G,
               const int32_t* __restrict__ mem_len, int m_cap, float qscale, int n_split,
               __nv_bfloat16* __restrict__ out, float* __restrict__ part_o,
               float2* __restrict__ part_ml, int* __restrict__ status) {
  using K = ACfg<D>;
  extern __shared__ __align__(1024) unsigned char smem_dyn[];
  __shared__ AAux aux;
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
  unsigned char* sQ = base;
  unsigned char* sKV = sQ + K::Q_BYTES;
  unsigned char* sP = sKV + kStages * K::STAGE;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int mt = blockIdx.x / n_split, sp = blockIdx.x % n_split;
  const int g = blockIdx.y, b = blockIdx.z;
  const int TQ = kRows / G;  // tokens per CTA
  const int tok0 = mt * TQ;
  const int n_tok = min(TQ, T - tok0);
  const int M = min(max(mem_len[b], 0), m_cap);
  const int lim_max = T_loc - T + tok0 + n_tok - 1;  // last local key any row sees
  const int n_mt = (M + kKeys - 1) / kKeys;
  const int n_lt = (lim_max + 1 + kKeys - 1) / kKeys;
  const int nt_all = n_mt + n_lt;
  // this CTA's share [j_lo, j_hi) of the key tiles
  const int j_lo = (int)((int64_t)sp * nt_all / n_split);
  const int j_hi = (int)((int64_t)(sp + 1) * nt_all / n_split);
  if (j_lo == j_hi) {  // nothing to attend: an empty partial (uniform exit)
    for (int r = threadIdx.x; r < kRows; r += blockDim.x) {
      if (r / G >= n_tok) continue;
      const int64_t row_id = ((int64_t)b * Hq + g * G + r % G) * T + tok0 + r / G;
      float* po = part_o + (row_id * n_split + sp) * D;
      for (int d = 0; d < D; ++d) po[d] = 0.f;
      part_ml[row_id * n_split + sp] = make_float2(-INFINITY, 0.f);
    }
    return;
  }
  const int nt = j_hi - j_lo;  // tiles j_lo + 0 .. j_lo + nt - 1

  if (threadIdx.x == 0) {
    tc::mbar_init(&aux.q_full, 1);
    for (int i = 0; i < kStages; ++i) {
      tc::mbar_init(&aux.kv_full[i], 1);
      tc::mbar_init(&aux.kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&aux.s_full[i], 1);
      tc::mbar_init(&aux.s_empty[i], kSoftWarps);
      tc::mbar_init(&aux.p_full[i], kSoftWarps);
    }
    tc::mbar_init(&aux.o_full, 1);
    aux.abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(&aux.tmem_base, K::TMEM_COLS);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = aux.tmem_base;
  const uint32_t tS[2] = {tmem, tmem + kKeys};
  const uint32_t tO = tmem + 2 * kKeys;
  volatile int* abort_flag = &aux.abort_flag;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t issued = 0;
      tc::mbar_arrive_expect_tx(&aux.q_full, K::Q_BYTES);
#pragma unroll
      for (int kb = 0; kb < K::KB; ++kb)
        tc::tma_load_3d(sQ + kb * kRows * 128, &tm_q, &aux.q_full, kb * 64, g * G,
                        b * T + tok0);
      for (int j = 0; j < nt; ++j) {
        const int st = j % kStages;
        if (*abort_flag || !tc::mbar_wait(&aux.kv_empty[st], ((j / kStages) & 1) ^ 1)) {
          record_error(status, MSA_ERR_TIMEOUT);
          *abort_flag = 1;
          break;
        }
        unsigned char* k_dst = sKV + st * K::STAGE;
        unsigned char* v_dst = k_dst + K::K_BYTES;
        tc::mbar_arrive_expect_tx(&aux.kv_full[st], K::STAGE);
        const int jj = j_lo + j;
        const bool mem = jj < n_mt;
        const CUtensorMap* mk = mem ? &tm_km : &tm_kl;
        const CUtensorMap* mv = mem ? &tm_vm : &tm_vl;
        const int row = mem ? b * m_cap + jj * kKeys : b * T_loc + (jj - n_mt) * kKeys;
#pragma unroll
        for (int kb = 0; kb < K::KB; ++kb) {
          tc::tma_load_3d(k_dst + kb * kKeys * 128, mk, &aux.kv_full[st], kb * 64, g, row);
          tc::tma_load_3d(v_dst + kb * kKeys * 128, mv, &aux.kv_full[st], kb * 64, g, row);
        }
        ++issued;
      }
      // every load issued must land before the CTA exits
      tc::mbar_wait(&aux.q_full, 0);
      for (uint32_t v = issued > (uint32_t)kStages ? issued - kStages : 0; v < issued; ++v)
        tc::mbar_wait(&aux.kv_full[v % kStages], (v / kStages) & 1);
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      const uint32_t q0 = tc::smem_u32(sQ);
      auto fail = [&]() {
        record_error(status, MSA_ERR_TIMEOUT);
        *abort_flag = 1;
      };
      auto issue_s = [&](int j) -> bool {
        const int st = j % kStages, sb = j & 1;
        if (*abort_flag || !tc::mbar_wait(&aux.kv_full[st], (j / kStages) & 1) ||
            !tc::mbar_wait(&aux.s_empty[sb], ((j >> 1) & 1) ^ 1))
          return false;
        tc::tc_fence_after();
        const uint32_t k0 = tc::smem_u32(sKV + st * K::STAGE);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (kRows * 128) + (kk & 3) * 32;
          const uint32_t koff = (kk >> 2) * (kKeys * 128) + (kk & 3) * 32;
          tc::mma_bf16_ss(tS[sb], tc::sdesc_kmajor_sw128(q0 + off),
                          tc::sdesc_kmajor_sw128(k0 + koff), K::IDESC_S, kk > 0 ? 1u : 0u);
        }
        tc::mma_commit(&aux.s_full[sb]);
        return true;
      };
      auto issue_pv = [&](int j) -> bool {
        const int st = j % kStages, pb = j & 1;
        // P of tile j written (and any rescale of O done) by the softmax
        if (*abort_flag || !tc::mbar_wait(&aux.p_full[pb], (j >> 1) & 1)) return false;
        tc::tc_fence_after();
        const uint32_t p0 = tc::smem_u32(sP + pb * K::P_BYTES);
        const uint32_t v0 = tc::smem_u32(sKV + st * K::STAGE + K::K_BYTES);
#pragma unroll
        for (int kk = 0; kk < kKeys / 16; ++kk) {
          // A = P (rows x keys, K-major, 64-key blocks); B = V (keys x d,
          // MN-major: 64-d column blocks 128*128 B apart, 16 keys = 2048 B)
          const uint32_t poff = (kk >> 2) * (kRows * 128) + (kk & 3) * 32;
          tc::mma_bf16_ss(tO, tc::sdesc_kmajor_sw128(p0 + poff),
                          sdesc_mnmajor_sw128(v0 + kk * 16 * 128, kKeys * 128), K::IDESC_O,
                          (j > 0 || kk > 0) ? 1u : 0u);
        }
        tc::mma_commit(&aux.o_full);
        tc::mma_commit(&aux.kv_empty[st]);
        return true;
      };
      if (!tc::mbar_wait(&aux.q_full, 0)) fail();
      else if (nt > 0) {
        bool ok = issue_s(0);
        for (int j = 0; ok && j < nt; ++j) {
          if (j + 1 < nt) ok = issue_s(j + 1);
          if (ok) ok = issue_pv(j);
        }
        if (!ok) fail();
      }
    }
  } else {
    // ------------------------------------------------------------- softmax
    // One thread per query row.  O accumulates in TMEM across key tiles;
    // the row's reference maximum m_run only moves when a tile's maximum
    // exceeds it by more than 2^kRescaleLog2 -- then O (in TMEM) and l are
    // rescaled once, after the previous P V has landed -- so p = 2^(s - m_run)
    // stays <= 2^kRescaleLog2 and most tiles need no rescale at all.
    constexpr float kRescaleLog2 = 8.f;
    const int quad = warp & 3;
    const int r = quad * 32 + lane;  // this thread's query row (TMEM lane)
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    const int tok = tok0 + r / G;
    const int lim = T_loc - T + tok;  // last visible local key
    float m_run = -INFINITY, l_run = 0.f;
    auto wait_o = [&](int j) {  // the P V of tile j has completed
      if (!*abort_flag && !tc::mbar_wait(&aux.o_full, j & 1)) {
        record_error(status, MSA_ERR_TIMEOUT);
        *abort_flag = 1;
      }
      tc::tc_fence_after();
    };
    for (int j = 0; j < nt; ++j) {
      const int sb = j & 1;
      if (!*abort_flag && !tc::mbar_wait(&aux.s_full[sb], (j >> 1) & 1)) {
        record_error(status, MSA_ERR_TIMEOUT);
        *abort_flag = 1;
      }
      tc::tc_fence_after();
      // visible keys of this tile: memory rows < M, local rows <= lim
      const int jj = j_lo + j;
      const bool mem = jj < n_mt;
      const int key0 = mem ? jj * kKeys : (jj - n_mt) * kKeys;
      const int n_vis = mem ? min(kKeys, M - key0) : max(0, min(kKeys, lim - key0 + 1));
      uint32_t sv[kKeys];
#pragma unroll
      for (int c = 0; c < kKeys / 32; ++c)
        tc::tmem_ld32(tS[sb] + lane_addr + c * 32, *reinterpret_cast<uint32_t(*)[32]>(sv + c * 32));
      tc::tmem_ld_wait();
      float mraw = -INFINITY;  // raw (unscaled) maximum of the visible scores
#pragma unroll
      for (int i = 0; i < kKeys; ++i)
        if (i < n_vis) mraw = fmaxf(mraw, __uint_as_float(sv[i]));
      const float mt = mraw * qscale;  // qscale > 0 keeps the order
      // rows whose maximum grew too much rescale O and l (warp-collective)
      const bool grow = mt > m_run + kRescaleLog2;
      float alpha = 1.f;
      if (grow) {
        alpha = m_run == -INFINITY ? 0.f : ex2_approx(m_run - mt);
        m_run = mt;
      }
      if (__any_sync(0xffffffffu, grow && alpha != 0.f) && j > 0) {
        wait_o(j - 1);
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t v[32];
          tc::tmem_ld32(tO + lane_addr + c * 32, v);
          tc::tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * alpha);
          tmem_st32(tO + lane_addr + c * 32, v);
        }
        tmem_st_wait();
      }
      l_run *= alpha;
      // p = 2^(s*qscale - m_run) as bf16 into the swizzled P tile
      unsigned char* prow = sP + sb * K::P_BYTES + r * 128;
      const float neg_m = m_run == -INFINITY ? 0.f : -m_run;
      float ls = 0.f;
#pragma unroll
      for (int c = 0; c < kKeys / 32; ++c) {
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const int k0 = c * 32 + i;
          const float p0 = k0 < n_vis ? ex2_approx(fmaf(__uint_as_float(sv[k0]), qscale, neg_m)) : 0.f;
          const float p1 =
              k0 + 1 < n_vis ? ex2_approx(fmaf(__uint_as_float(sv[k0 + 1]), qscale, neg_m)) : 0.f;
          ls += p0 + p1;
          w[i / 2] = pack_bf16(p0, p1);
        }
        // keys c*32 .. c*32+31 are 16-byte pieces 4(c%2) .. 4(c%2)+3 of K
        // block c/2 of row r, stored at their 128B-swizzled positions
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int piece = (c & 1) * 4 + q;
          *reinterpret_cast<uint4*>(prow + (c >> 1) * (kRows * 128) + ((piece ^ (r & 7)) << 4)) =
              make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
        }
      }
      l_run += ls;
      if (mem && M - key0 < kKeys && r >= M - key0) {
        // rows past mem_len in the last memory tile hold whatever the
        // caller's buffer holds there; zero their V so that 0 * V stays 0
        unsigned char* vrow = sKV + (j % kStages) * K::STAGE + K::K_BYTES + r * 128;
#pragma unroll
        for (int kb = 0; kb < K::KB; ++kb)
#pragma unroll
          for (int q = 0; q < 8; ++q)
            *reinterpret_cast<uint4*>(vrow + kb * (kKeys * 128) + q * 16) = make_uint4(0, 0, 0, 0);
      }
      tc::fence_proxy_async_smem();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        tc::mbar_arrive(&aux.p_full[sb]);
        tc::mbar_arrive(&aux.s_empty[sb]);
      }
    }
    // the last P V, then this row's output.  s_full of tile nt-1 implied
    // that P V nt-3 had completed; wait for nt-2 and nt-1 in turn, so that
    // each parity wait is at most one phase behind.
    if (nt >= 2) wait_o(nt - 2);
    wait_o(nt - 1);
    const bool row_ok = r / G < n_tok;
    const int64_t row_id = ((int64_t)b * Hq + g * G + r % G) * T + tok;
    const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t v[32];
      tc::tmem_ld32(tO + lane_addr + c * 32, v);
      tc::tmem_ld_wait();
      if (!row_ok) continue;
      if (n_split > 1) {
        float* po = part_o + (row_id * n_split + sp) * D + c * 32;
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          *reinterpret_cast<float4*>(po + i) =
              make_float4(__uint_as_float(v[i]), __uint_as_float(v[i + 1]),
                          __uint_as_float(v[i + 2]), __uint_as_float(v[i + 3]));
      } else {
        __nv_bfloat16* op = out + (((int64_t)b * T + tok) * Hq + g * G + r % G) * D + c * 32;
#pragma unroll
        for (int i = 0; i < 32; i += 8)
          *reinterpret_cast<uint4*>(op + i) = make_uint4(
              pack_bf16(__uint_as_float(v[i]) * inv, __uint_as_float(v[i + 1]) * inv),
              pack_bf16(__uint_as_float(v[i + 2]) * inv, __uint_as_float(v[i + 3]) * inv),
              pack_bf16(__uint_as_float(v[i + 4]) * inv, __uint_as_float(v[i + 5]) * inv),
              pack_bf16(__uint_as_float(v[i + 6]) * inv, __uint_as_float(v[i + 7]) * inv));
      }
    }
    if (row_ok && n_split > 1) part_ml[row_id * n_split + sp] = make_float2(m_run, l_run);
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, K::TMEM_COLS);
  }
}

// Global RoPE of the query and the local keys, one launch: CTA i owns local
// positions [i*kPosPerCta, ...): it builds their (cos, sin) in shared memory
// (angles reduced in double), then rotates every local K row and every query
// row at those positions (query token t sits at local position T_loc - T + t)
// with 16-byte loads of an element group and its rotate-half partner.
constexpr int kPosPerCta = 4;

template <int D>
__global__ void __launch_bounds__(256)
rope_prep_kernel(int B, int T, int T_loc, int Hq, int H, int64_t pos0, double base,
                 const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k_loc,
                 __nv_bfloat16* __restrict__ q_rot, __nv_bfloat16* __restrict__ k_rot) {
  constexpr int HALF = D / 2;
  constexpr int UPH = HALF / 8;  // 16-byte pair units per head
  __shared__ float2 cs[kPosPerCta][HALF];
  const int p0 = blockIdx.x * kPosPerCta;
  const int np = min(kPosPerCta, T_loc - p0);
  for (int e = threadIdx.x; e < np * HALF; e += blockDim.x) {
    const int j = e / HALF, i = e % HALF;
    cs[j][i] = rope_cs(pos0 + p0 + j, rope_inv_freq(base, i, D));
  }
  __syncthreads();
  // local keys: B x np positions x H heads x UPH units
  const int nk = B * np * H * UPH;
  for (int e = threadIdx.x; e < nk; e += blockDim.x) {
    const int u = e % UPH, h = (e / UPH) % H, j = (e / (UPH * H)) % np, b = e / (UPH * H * np);
    const int64_t off = (((int64_t)b * T_loc + p0 + j) * H + h) * D + u * 8;
    float x1[8], x2[8], y1[8], y2[8];
    Vec16<__nv_bfloat16>::unpack(ldg16(k_loc + off), x1);
    Vec16<__nv_bfloat16>::unpack(ldg16(k_loc + off + HALF), x2);
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      const float2 c = cs[j][u * 8 + t];
      y1[t] = x1[t] * c.x - x2[t] * c.y;
      y2[t] = x2[t] * c.x + x1[t] * c.y;
    }
    st16(k_rot + off, Vec16<__nv_bfloat16>::pack(y1));
    st16(k_rot + off + HALF, Vec16<__nv_bfloat16>::pack(y2));
  }
  // query tokens at these positions
  const int first_q = T_loc - T;  // local position of query token 0
  const int t_lo = max(p0, first_q) - first_q, t_hi = p0 + np - first_q;
  if (t_hi <= t_lo) return;
  const int nt = t_hi - t_lo;
  const int nq = B * nt * Hq * UPH;
  for (int e = threadIdx.x; e < nq; e += blockDim.x) {
    const int u = e % UPH, h = (e / UPH) % Hq, tt = (e / (UPH * Hq)) % nt,
              b = e / (UPH * Hq * nt);
    const int t = t_lo + tt;
    const int j = first_q + t - p0;
    const int64_t off = (((int64_t)b * T + t) * Hq + h) * D + u * 8;
    float x1[8], x2[8], y1[8], y2[8];
    Vec16<__nv_bfloat16>::unpack(ldg16(q + off), x1);
    Vec16<__nv_bfloat16>::unpack(ldg16(q + off + HALF), x2);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float2 c = cs[j][u * 8 + i];
      y1[i] = x1[i] * c.x - x2[i] * c.y;
      y2[i] = x2[i] * c.x + x1[i] * c.y;
    }
    st16(q_rot + off, Vec16<__nv_bfloat16>::pack(y1));
    st16(q_rot + off + HALF, Vec16<__nv_bfloat16>::pack(y2));
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    else
      cudaGetLastError();
  }
  return fn;
}

// bf16 [rows][heads][D] viewed as dims {D, heads, rows}; box {64, bh, br}.
bool map3(CUtensorMap* m, const void* ptr, int D, int heads, int64_t rows, int bh, int br) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)heads, (cuuint64_t)rows};
  const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)heads * D * 2};
  const cuuint32_t box[3] = {64, (cuuint32_t)bh, (cuuint32_t)br};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct TcPlan {
  int n_split;
  size_t q_bytes, k_bytes, po_bytes, ml_bytes, total;
};

// Key-tile splits: enough CTAs to cover the SMs twice, at most 3 (each split
// re-reads the query tile and writes an fp32 partial) and at most the
// number of key tiles.
TcPlan tc_plan(int B, int T, int T_loc, int Hq, int H, int D, int m_cap) {
  TcPlan p{};
  const int G = Hq / H;
  const int TQ = kRows / G;
  const int64_t base = (int64_t)((T + TQ - 1) / TQ) * H * B;
  const int64_t max_tiles = (m_cap + kKeys - 1) / kKeys + (T_loc + kKeys - 1) / kKeys;
  int64_t ns = (2LL * num_sms() + base - 1) / base;
  ns = std::min<int64_t>(ns, 3);
  ns = std::min<int64_t>(ns, max_tiles);
  p.n_split = (int)std::max<int64_t>(ns, 1);
  p.q_bytes = round_up((size_t)B * T * Hq * D * 2, 256);
  p.k_bytes = round_up((size_t)B * T_loc * H * D * 2, 256);
  const size_t rows = (size_t)B * Hq * T;
  p.po_bytes = p.n_split > 1 ? round_up(rows * p.n_split * D * sizeof(float), 256) : 0;
  p.ml_bytes = p.n_split > 1 ? round_up(rows * p.n_split * sizeof(float2), 256) : 0;
  p.total = p.q_bytes + p.k_bytes + p.po_bytes + p.ml_bytes;
  return p;
}

template <int D>
int launch_tc(int B, int T, int T_loc, int Hq, int H, const void* q, const void* k_mem,
              const void* v_mem, const int32_t* mem_len, int m_cap, const void* k_loc,
              const void* v_loc, int pos0, float rope_base, float qscale, void* out, void* ws,
              cudaStream_t s) {
  using K = ACfg<D>;
  const int G = Hq / H;
  const TcPlan p = tc_plan(B, T, T_loc, Hq, H, D, m_cap);
  unsigned char* w = static_cast<unsigned char*>(ws);
  __nv_bfloat16* q_rot = reinterpret_cast<__nv_bfloat16*>(w);
  __nv_bfloat16* k_rot = reinterpret_cast<__nv_bfloat16*>(w + p.q_bytes);
  float* part_o = reinterpret_cast<float*>(w + p.q_bytes + p.k_bytes);
  float2* part_ml = reinterpret_cast<float2*>(w + p.q_bytes + p.k_bytes + p.po_bytes);
  rope_prep_kernel<D><<<(unsigned)((T_loc + kPosPerCta - 1) / kPosPerCta), 256, 0, s>>>(
      B, T, T_loc, Hq, H, pos0, (double)rope_base, static_cast<const __nv_bfloat16*>(q),
      static_cast<const __nv_bfloat16*>(k_loc), q_rot, k_rot);
  int rc = check_launch();
  if (rc) return rc;

  CUtensorMap tq, tkm, tvm, tkl, tvl;
  const int TQ = kRows / G;
  const int64_t mem_rows = std::max<int64_t>((int64_t)B * m_cap, 1);
  const void* km = m_cap > 0 ? k_mem : k_rot;  // any valid address when there is no memory
  const void* vm = m_cap > 0 ? v_mem : v_loc;
  if (!map3(&tq, q_rot, D, Hq, (int64_t)B * T, G, TQ) ||
      !map3(&tkm, km, D, H, m_cap > 0 ? mem_rows : (int64_t)B * T_loc, 1, kKeys) ||
      !map3(&tvm, vm, D, H, m_cap > 0 ? mem_rows : (int64_t)B * T_loc, 1, kKeys) ||
      !map3(&tkl, k_rot, D, H, (int64_t)B * T_loc, 1, kKeys) ||
      !map3(&tvl, v_loc, D, H, (int64_t)B * T_loc, 1, kKeys))
    return note_cuda(cudaErrorInvalidValue);
  auto kern = attn_tc_kernel<D>;
  rc = ensure_smem_attr(reinterpret_cast<const void*>(kern), (int)K::SMEM);
  if (rc) return rc;
  const dim3 grid((unsigned)((T + TQ - 1) / TQ * p.n_split), (unsigned)H, (unsigned)B);
  kern<<<grid, kThreads, K::SMEM, s>>>(tq, tkm, tvm, tkl, tvl, T, T_loc, Hq, H, G, mem_len,
                                       m_cap, qscale, p.n_split, static_cast<__nv_bfloat16*>(out),
                                       part_o, part_ml, device_status_ptr());
  rc = check_launch();
  if (rc || p.n_split == 1) return rc;
  return attn_combine_bf16(B, T, Hq, D, p.n_split, part_o, part_ml, out, s);
}

}  // namespace

bool attn_tc_supported(int B, int T, int T_loc, int Hq, int H, int D, int m_cap) {
  if (T < 2 || (D != 64 && D != 128) || H <= 0 || Hq % H) return false;
  const int G = Hq / H;
  if (G > 16 || (G & (G - 1))) return false;
  if ((int64_t)B * T > (1LL << 30) || (int64_t)B * T_loc > (1LL << 30) ||
      (int64_t)B * m_cap > (1LL << 30) || B > 65535 || H > 65535)
    return false;
  return true;
}

size_t attn_tc_workspace_size(int B, int T, int T_loc, int Hq, int H, int D, int m_cap) {
  return tc_plan(B, T, T_loc, Hq, H, D, m_cap).total;
}

int attn_tc_launch(int B, int T, int T_loc, int Hq, int H, int D, const void* q,
                   const void* k_mem, const void* v_mem, const int32_t* mem_len, int m_cap,
                   const void* k_loc, const void* v_loc, int pos0, float rope_base, float qscale,
                   void* out, void* ws, cudaStream_t s) {
  if (!aligned16(q) || !aligned16(k_loc) || !aligned16(v_loc) || !aligned16(out) ||
      (m_cap > 0 && (!aligned16(k_mem) || !aligned16(v_mem))))
    return MSA_ERR_INVALID_ARG;
  if (D == 64)
    return launch_tc<64>(B, T, T_loc, Hq, H, q, k_mem, v_mem, mem_len, m_cap, k_loc, v_loc, pos0,
                         rope_base, qscale, out, ws, s);
  return launch_tc<128>(B, T, T_loc, Hq, H, q, k_mem, v_mem, mem_len, m_cap, k_loc, v_loc, pos0,
                        rope_base, qscale, out, ws, s);
}

}  // namespace msa
