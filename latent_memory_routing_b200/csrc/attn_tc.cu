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
//   * attn_tc_kernel: a persistent grid, one CTA per SM, working through
//     items of (two Q tiles of 128 rows, KV head, batch, key split), claimed
//     at run time in groups of (batch, KV head) pairs whose keys and values
//     fit a share of the L2, heaviest first within a group (causal work
//     grows with the query block).
//     An item's Q tiles and first K/V tiles load while the previous item's
//     last tiles are still in the tensor core and softmax, and its O is read
//     out of TMEM before the stores, so the next item's MMAs start at once:
//     a CTA's setup, first-load latency and epilogue are paid once per SM
//     instead of once per item.  Up to 3 splits of the key tiles, at most one
//     per 8 tiles, are merged by the split-KV combine kernel when there are
//     too few query blocks to fill the SMs.  GQA rows are packed as (token,
//     head of the group): a TMA box of {64 d, G heads, 128/G tokens} lands as
//     128 rows of 128 B -- a Q tile of all G query heads sharing one KV head.
//     Key tiles of 128 rows come first from the memory (mem_len rows, clamped
//     to [0, m_cap]) then from the local context (up to the block's last
//     visible key), each as K and V TMA boxes.
//     - warpgroup 0: warp 0 (one lane) loads the Q tiles, then runs a 2-stage
//       K/V ring; warp 1 (one lane) issues tcgen05.mma.  S_i = Q_i K^T
//       (M = 128, N = 128 keys, K = D) goes to the 128 TMEM columns of Q tile
//       i; O_i += P_i V (M = 128, N = D, K = 128 keys) reads P_i from those
//       same TMEM columns (the A operand in tensor memory) and V MN-major
//       straight from its TMA tile.  The issue order
//       S_0(0) S_1(0) | P_0V(0) S_0(1) P_1V(0) S_1(1) | ...
//       keeps one softmax warpgroup busy while the tensor core serves the
//       other;
//     - warpgroups 1 and 2 (one per Q tile, one thread per row, registers
//       moved to them by setmaxnreg): online softmax in fp32 -- the tile's
//       scores read once from TMEM, masked row maximum, p = 2^(s - m) (SFU
//       ex2) packed to bf16 and written back over S in TMEM, row sum.  O
//       accumulates in TMEM; a row rescales O and its sum only when its
//       maximum grows by more than 2^8 (then p <= 256 meanwhile), which after
//       the first tiles is rare.  In the last memory tile, warpgroup 1 zeroes
//       the V rows past mem_len in shared memory before P V reads them (in
//       the fused form, the rows of any group past its document's end).
//   * Every mbarrier wait is bounded; a timeout records MSA_ERR_TIMEOUT and
//     all roles finish their loops without waiting.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdlib>

#include "attn_tc.cuh"
#include "msa_common.cuh"
#include "tc_ptx.cuh"

namespace msa {
namespace {

constexpr int kRows = 128;   // query rows per Q tile (MMA M)
constexpr int kQT = 2;       // Q tiles per CTA, one softmax warpgroup each
constexpr int kKeys = 128;   // keys per tile (MMA N of S, K of P V)
constexpr int kSoftWarps = 4 * kQT;
// warpgroup 0: TMA producer (warp 0), MMA issuer (warp 1), two idle warps;
// warpgroups 1 .. kQT: softmax.  Registers move from warpgroup 0 to the
// softmax warpgroups: 128 x REG_LOW + 256 x REG_HIGH = 384 x 168, the
// block's launch allocation under __launch_bounds__(384, 1).
constexpr int kThreads = 128 + 32 * kSoftWarps;
constexpr int kStages = 2;

template <int D>
struct ACfg {
  static constexpr int KB = D / 64;
  static constexpr int Q_BYTES = KB * kRows * 128;   // one Q tile
  static constexpr int K_BYTES = KB * kKeys * 128;
  static constexpr int V_BYTES = KB * kKeys * 128;
  static constexpr int STAGE = K_BYTES + V_BYTES;
  static constexpr size_t SMEM = 1024 + kQT * Q_BYTES + kStages * STAGE;
  // TMEM: per Q tile an S tile (128 fp32 columns, whose first 64 columns
  // then hold P as packed bf16) and an O tile (D fp32 columns)
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(kQT * (kKeys + D) <= 512, "TMEM budget");
  // S: M=128, N=128 keys, A (Q) and B (K) K-major
  static constexpr uint32_t IDESC_S = tc::idesc_bf16_f32(kRows, kKeys);
  // O: M=128, N=D, A (P, TMEM) K-major, B (V) MN-major (bit 16)
  static constexpr uint32_t IDESC_O = tc::idesc_bf16_f32(kRows, D) | (1u << 16);
  // registers per thread of warpgroup 0 (producer, MMA issuer: the item
  // bookkeeping of the persistent loop) and of the softmax warpgroups,
  // chosen where the compiler reports no or few spills for either
  static constexpr int REG_LOW = D == 128 ? 72 : 88;
  static constexpr int REG_HIGH = D == 128 ? 216 : 208;
  // the fused form's producer also holds a memory tile's 16 group rows
  static constexpr int REG_LOW_FUSED = 88;
  static constexpr int REG_HIGH_FUSED = 208;
  static_assert(kQT == 2 && 128 * REG_LOW + 256 * REG_HIGH == 384 * 168, "register split");
  static_assert(128 * REG_LOW_FUSED + 256 * REG_HIGH_FUSED == 384 * 168, "register split");
};

// L2 budget of a group of (batch, KV head) pairs' key/value rows (of the
// 126 MB L2; the query tiles stream beside them)
constexpr int64_t kL2GroupBytes = 48ll << 20;

// item-id ring between the producer and the other roles
constexpr int kSched = 4;
constexpr int kSchedReaders = 1 + kSoftWarps;  // the MMA issuer, each softmax warp
// the producer claims the next item this many tiles before its current
// item's last tile load
constexpr int kClaimAhead = 3;

struct AAux {
  uint64_t q_full, q_empty, kv_full[kStages], kv_empty[kStages], s_full[kQT], p_full[kQT],
      o_full[kQT], o_empty[kQT], sched_full[kSched], sched_empty[kSched];
  int sched_id[kSched];
  uint32_t tmem_base;
  int abort_flag;
};

using tc::mma_bf16_ts;
using tc::sdesc_mnmajor_sw128;

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

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ unsigned long long f2_pack(float lo, float hi) {
  return (unsigned long long)__float_as_uint(lo) | ((unsigned long long)__float_as_uint(hi) << 32);
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Work item `idx` of a call: the (batch, KV head) pairs in groups of `pg`
// consecutive pairs, group after group; within a group heaviest first --
// query blocks in descending order (under a causal mask later blocks see
// more key tiles) -- then pair and key split.
struct Item {
  int mt, b, g, sp;
};
__device__ __forceinline__ Item item_of(int idx, int B, int H, int n_split, int n_qb, int pg) {
  const int P = B * H;                        // (batch, KV head) pairs
  const int per_group = n_qb * pg * n_split;  // items of a full group of pg pairs
  const int k = min(idx / per_group, P / pg);
  const int r = idx - k * per_group;
  const int per_qb = min(pg, P - k * pg) * n_split;
  Item it;
  it.mt = n_qb - 1 - r / per_qb;
  const int rem = r % per_qb;
  const int pair = k * pg + rem / n_split;
  it.b = pair / H;
  it.g = pair % H;
  it.sp = rem % n_split;
  return it;
}

// The key tiles of an item: the memory tiles (mem_len rows, clamped), then
// the local tiles up to the block's last visible key; the split owns
// [j_lo, j_lo + nt) of them.
struct Span {
  int tok0, n_tok, M, n_mt, j_lo, nt;
};
template <bool kFused>
__device__ __forceinline__ Span span_of(const Item& it, int T, int T_loc, int TQ,
                                        const int32_t* __restrict__ mem_len, int m_cap,
                                        int max_groups, int n_split) {
  Span s;
  s.tok0 = it.mt * kQT * TQ;
  s.n_tok = min(kQT * TQ, T - s.tok0);
  const int ml = max(__ldg(mem_len + it.b), 0);
  s.M = kFused ? 8 * min(ml, max_groups) : min(ml, m_cap);
  const int lim_max = T_loc - T + s.tok0 + s.n_tok - 1;  // last local key any row sees
  s.n_mt = (s.M + kKeys - 1) / kKeys;
  const int nt_all = s.n_mt + (lim_max + 1 + kKeys - 1) / kKeys;
  s.j_lo = (int)((int64_t)it.sp * nt_all / n_split);
  s.nt = (int)((int64_t)(it.sp + 1) * nt_all / n_split) - s.j_lo;
  return s;
}

// kFused: memory rows read straight from the pooled bank, per query a list
// of 8-row groups (first bank row, rows of the group inside its document)
// in rank order; tm_km / tm_vm map the bank with 8-row boxes (one
// 128B-swizzle atom), a memory tile is 16 groups, and `mem_len` holds the
// group count.  Rows past a document's end are other bank rows: masked, and
// their V zeroed in shared memory before P V reads it.
//
// Persistent: one CTA per SM (grid = min(items, SMs)); CTA c starts with
// item c and claims the next one from `next_item` (zeroed by the RoPE
// preparation) while the loads of its current item's last tile are issued.
// The producer publishes each item id in a shared-memory ring that the MMA
// issuer and the softmax warps read.  Every ring, tile and item barrier
// counts phases over the whole CTA lifetime: the K/V ring by the CTA's
// running tile count, q_full / q_empty / o_full / o_empty by its running
// count of non-empty items.
template <int D, bool kFused>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_km,
               const __grid_constant__ CUtensorMap tm_vm, const __grid_constant__ CUtensorMap tm_kl,
               const __grid_constant__ CUtensorMap tm_vl, int B, int T, int T_loc, int Hq, int H,
               int G, const int32_t* __restrict__ mem_len, int m_cap,
               const int2* __restrict__ groups, int max_groups, float qscale, int n_split,
               int n_qb, int n_items, int pairs_per_group, int* __restrict__ next_item,
               __nv_bfloat16* __restrict__ out, float* __restrict__ part_o,
               float2* __restrict__ part_ml, int* __restrict__ status) {
  using K = ACfg<D>;
  // launched as a programmatic dependent of the RoPE preparation: wait for
  // its completion (and the visibility of its writes, the zeroed item
  // counter among them) before reading anything
  pdl_wait();
  extern __shared__ __align__(1024) unsigned char smem_dyn[];
  __shared__ AAux aux;
  unsigned char* base = tc::smem_align<1024>(smem_dyn);
  unsigned char* sQ = base;                        // kQT Q tiles
  unsigned char* sKV = sQ + kQT * K::Q_BYTES;      // kStages x (K tile, V tile)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int TQ = kRows / G;  // tokens per Q tile

  if (threadIdx.x == 0) {
    tc::mbar_init(&aux.q_full, 1);
    tc::mbar_init(&aux.q_empty, 1);
    for (int i = 0; i < kStages; ++i) {
      tc::mbar_init(&aux.kv_full[i], 1);
      tc::mbar_init(&aux.kv_empty[i], 1);
    }
    for (int i = 0; i < kQT; ++i) {
      tc::mbar_init(&aux.s_full[i], 1);
      tc::mbar_init(&aux.p_full[i], 4);
      tc::mbar_init(&aux.o_full[i], 1);
      tc::mbar_init(&aux.o_empty[i], 4);
    }
    for (int i = 0; i < kSched; ++i) {
      tc::mbar_init(&aux.sched_full[i], 1);
      tc::mbar_init(&aux.sched_empty[i], kSchedReaders);
    }
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
  // TMEM columns: S/P of tile i at i*kKeys, O of tile i at kQT*kKeys + i*D
  volatile int* abort_flag = &aux.abort_flag;
  auto fail = [&]() {
    record_error(status, MSA_ERR_TIMEOUT);
    *abort_flag = 1;
  };
  auto span = [&](const Item& it) {
    return span_of<kFused>(it, T, T_loc, TQ, mem_len, m_cap, max_groups, n_split);
  };

  if (warp < 4) {
   asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n"
                ::"n"(kFused ? K::REG_LOW_FUSED : K::REG_LOW));
   if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t tiles = 0, q_loads = 0;  // loads issued over the CTA's items
      int idx = blockIdx.x;
      bool ok = true;
      for (uint32_t n = 0; ok; ++n) {
        const int slot = n % kSched;
        if (*abort_flag || !tc::mbar_wait(&aux.sched_empty[slot], ((n / kSched) & 1) ^ 1)) {
          ok = false;
          break;
        }
        const bool live = idx < n_items;
        aux.sched_id[slot] = live ? idx : -1;
        tc::mbar_arrive(&aux.sched_full[slot]);  // release: the id is visible to the waiters
        if (!live) break;
        const Item it = item_of(idx, B, H, n_split, n_qb, pairs_per_group);
        const Span sp = span(it);
        int nxt = n_items;
        if (sp.nt == 0) {
          idx = atomicAdd(next_item, 1) + (int)gridDim.x;
          continue;
        }
        // the Q tiles are free once the previous item's last S has completed
        if (q_loads > 0 && (*abort_flag || !tc::mbar_wait(&aux.q_empty, (q_loads - 1) & 1))) {
          ok = false;
          break;
        }
        tc::mbar_arrive_expect_tx(&aux.q_full, kQT * K::Q_BYTES);
#pragma unroll
        for (int i = 0; i < kQT; ++i)
#pragma unroll
          for (int kb = 0; kb < K::KB; ++kb)
            tc::tma_load_3d(sQ + i * K::Q_BYTES + kb * kRows * 128, &tm_q, &aux.q_full, kb * 64,
                            it.g * G, it.b * T + sp.tok0 + i * TQ);
        ++q_loads;
        const int2* gq = kFused ? groups + (int64_t)it.b * max_groups : nullptr;
        const int j_claim = max(sp.nt - kClaimAhead, 0);
        for (int j = 0; j < sp.nt; ++j) {
          // claim the next item a few tiles before this one's loads end
          if (j == j_claim) nxt = atomicAdd(next_item, 1) + (int)gridDim.x;
          const int st = tiles % kStages;
          const int jj = sp.j_lo + j;
          const bool mem = jj < sp.n_mt;
          // fused memory tile: its 16 groups' first bank rows, all read before
          // the slot wait (one round trip, overlapping it; the TMA issue below
          // is ordered after every memory access, so a read between two issues
          // would cost a round trip per group); past the last group, the last
          // one again (finite rows, masked) so every row of the tile is written
          int src[kKeys / 8];
          if (kFused && mem) {
            const int ng = sp.M / 8, g0 = jj * (kKeys / 8);
#pragma unroll
            for (int gi = 0; gi < kKeys / 8; ++gi) src[gi] = __ldg(&gq[min(g0 + gi, ng - 1)].x);
          }
          if (*abort_flag || !tc::mbar_wait(&aux.kv_empty[st], ((tiles / kStages) & 1) ^ 1)) {
            ok = false;
            break;
          }
          if (j == j_claim && nxt < n_items) {
            // its Q tiles into L2: the Q buffer frees only when this item's
            // last S completes, and from L2 the reload is short
            const Item ni = item_of(nxt, B, H, n_split, n_qb, pairs_per_group);
#pragma unroll
            for (int i = 0; i < kQT; ++i)
#pragma unroll
              for (int kb = 0; kb < K::KB; ++kb)
                tc::tma_prefetch_l2_3d(&tm_q, kb * 64, ni.g * G,
                                       ni.b * T + ni.mt * kQT * TQ + i * TQ);
          }
          unsigned char* k_dst = sKV + st * K::STAGE;
          unsigned char* v_dst = k_dst + K::K_BYTES;
          tc::mbar_arrive_expect_tx(&aux.kv_full[st], K::STAGE);
          const CUtensorMap* mk = mem ? &tm_km : &tm_kl;
          const CUtensorMap* mv = mem ? &tm_vm : &tm_vl;
          if (kFused && mem) {
            // 16 groups of 8 bank rows
#pragma unroll
            for (int gi = 0; gi < kKeys / 8; ++gi)
#pragma unroll
              for (int kb = 0; kb < K::KB; ++kb) {
                tc::tma_load_3d(k_dst + kb * kKeys * 128 + gi * 1024, mk, &aux.kv_full[st],
                                kb * 64, it.g, src[gi]);
                tc::tma_load_3d(v_dst + kb * kKeys * 128 + gi * 1024, mv, &aux.kv_full[st],
                                kb * 64, it.g, src[gi]);
              }
          } else {
            const int row =
                mem ? it.b * m_cap + jj * kKeys : it.b * T_loc + (jj - sp.n_mt) * kKeys;
#pragma unroll
            for (int kb = 0; kb < K::KB; ++kb) {
              tc::tma_load_3d(k_dst + kb * kKeys * 128, mk, &aux.kv_full[st], kb * 64, it.g,
                              row);
              tc::tma_load_3d(v_dst + kb * kKeys * 128, mv, &aux.kv_full[st], kb * 64, it.g,
                              row);
            }
          }
          ++tiles;
        }
        idx = nxt;
      }
      if (!ok) fail();
      // every load issued must land before the CTA exits
      if (q_loads > 0) tc::mbar_wait(&aux.q_full, (q_loads - 1) & 1);
      for (uint32_t v = tiles > (uint32_t)kStages ? tiles - kStages : 0; v < tiles; ++v)
        tc::mbar_wait(&aux.kv_full[v % kStages], (v / kStages) & 1);
    }
   } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    // order within an item: S_0(0) S_1(0) | P_0V(0) S_0(1) P_1V(0) S_1(1) |
    // ... so each softmax warpgroup works while the tensor core serves the
    // other one; S_i(j) is issued after P_iV(j-1), which makes the TMEM
    // columns that held P_i(j-1) safe to overwrite and lets s_full_i(j)
    // imply that P_iV(j-1) has completed.  The next item's S_i(0) follows
    // this item's last P_iV the same way; its first P_iV (which overwrites
    // O_i) waits until softmax group i has read this item's O_i out.
    if (lane == 0) {
      uint32_t tiles = 0, ne = 0;  // tiles and non-empty items so far
      bool ok = true;
      for (uint32_t n = 0; ok; ++n) {
        const int slot = n % kSched;
        if (*abort_flag || !tc::mbar_wait(&aux.sched_full[slot], (n / kSched) & 1)) {
          ok = false;
          break;
        }
        const int idx = aux.sched_id[slot];
        tc::mbar_arrive(&aux.sched_empty[slot]);
        if (idx < 0) break;
        const int nt = span(item_of(idx, B, H, n_split, n_qb, pairs_per_group)).nt;
        if (nt == 0) continue;
        ok = !*abort_flag && tc::mbar_wait(&aux.q_full, ne & 1);
        auto issue_s = [&](int i, int j) -> bool {
          const uint32_t v = tiles + j;
          const int st = v % kStages;
          if (*abort_flag || !tc::mbar_wait(&aux.kv_full[st], (v / kStages) & 1)) return false;
          // S_i(j) overwrites P_i(j-1); the P V that reads it was issued
          // (after its p_full wait) before this MMA, and the tensor core runs
          // one thread's MMAs in issue order
          tc::tc_fence_after();
          const uint64_t qd = tc::sdesc_kmajor_sw128(tc::smem_u32(sQ + i * K::Q_BYTES));
          const uint64_t kd = tc::sdesc_kmajor_sw128(tc::smem_u32(sKV + st * K::STAGE));
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * (kRows * 128) + (kk & 3) * 32;
            const uint32_t koff = (kk >> 2) * (kKeys * 128) + (kk & 3) * 32;
            tc::mma_bf16_ss(tmem + i * kKeys, tc::desc_add(qd, off), tc::desc_add(kd, koff),
                            K::IDESC_S, kk > 0 ? 1u : 0u);
          }
          tc::mma_commit(&aux.s_full[i]);
          // the item's last S: its Q tiles may be overwritten once it completes
          if (i == kQT - 1 && j == nt - 1) tc::mma_commit(&aux.q_empty);
          return true;
        };
        auto issue_pv = [&](int i, int j) -> bool {
          const uint32_t v = tiles + j;
          const int st = v % kStages;
          // O_i of the previous item read out of TMEM by softmax group i
          if (j == 0 && ne > 0 &&
              (*abort_flag || !tc::mbar_wait(&aux.o_empty[i], (ne - 1) & 1)))
            return false;
          // P_i(j) written (and any rescale of O_i done) by softmax group i
          if (*abort_flag || !tc::mbar_wait(&aux.p_full[i], v & 1)) return false;
          tc::tc_fence_after();
          const uint64_t vd =
              sdesc_mnmajor_sw128(tc::smem_u32(sKV + st * K::STAGE + K::K_BYTES), kKeys * 128);
#pragma unroll
          for (int kk = 0; kk < kKeys / 16; ++kk)
            mma_bf16_ts(tmem + kQT * kKeys + i * D, tmem + i * kKeys + kk * 8,
                        tc::desc_add(vd, kk * 16 * 128), K::IDESC_O, (j > 0 || kk > 0) ? 1u : 0u);
          if (j == nt - 1) tc::mma_commit(&aux.o_full[i]);  // O_i of the item final
          if (i == kQT - 1) tc::mma_commit(&aux.kv_empty[st]);
          return true;
        };
        for (int i = 0; ok && i < kQT; ++i) ok = issue_s(i, 0);
        for (int j = 0; ok && j < nt; ++j)
          for (int i = 0; ok && i < kQT; ++i) {
            ok = issue_pv(i, j);
            if (ok && j + 1 < nt) ok = issue_s(i, j + 1);
          }
        tiles += nt;
        ++ne;
      }
      if (!ok) fail();
    }
   }
  } else {
    // ------------------------------------------------------------- softmax
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n"
                 ::"n"(kFused ? K::REG_HIGH_FUSED : K::REG_HIGH));
    // Warpgroup i owns Q tile i, one thread per query row.  O_i accumulates
    // in TMEM; the row's reference maximum m_run only moves when a tile's
    // maximum exceeds it by more than 2^kRescaleLog2 -- then O_i (in TMEM)
    // and l are rescaled once (s_full_i(j) implies P_iV(j-1) is done) -- so
    // p = 2^(s - m_run) stays <= 2^kRescaleLog2 and most tiles need no
    // rescale.  P goes back into the S tile's first 64 TMEM columns as
    // packed bf16, the A operand of the P V MMA.
    constexpr float kRescaleLog2 = 8.f;
    const int qt = (warp - 4) >> 2;   // Q tile of this warpgroup
    const int quad = warp & 3;        // TMEM lane quarter
    const int r = quad * 32 + lane;   // row within the Q tile
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    const uint32_t tSP = tmem + qt * kKeys + lane_addr;
    const uint32_t tOi = tmem + kQT * kKeys + qt * D + lane_addr;
    uint32_t tiles = 0, ne = 0;  // tiles and non-empty items so far
    for (uint32_t n = 0;; ++n) {
      const int slot = n % kSched;
      if (*abort_flag) break;
      if (!tc::mbar_wait(&aux.sched_full[slot], (n / kSched) & 1)) {
        fail();
        break;
      }
      const int idx = aux.sched_id[slot];
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&aux.sched_empty[slot]);
      if (idx < 0) break;
      const Item it = item_of(idx, B, H, n_split, n_qb, pairs_per_group);
      const Span sp = span(it);
      const int tok_local = qt * TQ + r / G;
      const int tok = sp.tok0 + tok_local;
      const bool row_ok = tok_local < sp.n_tok;
      const int64_t row_id = ((int64_t)it.b * Hq + it.g * G + r % G) * T + tok;
      if (sp.nt == 0) {  // nothing to attend: an empty partial
        if (row_ok) {
          float* po = part_o + (row_id * n_split + it.sp) * D;
          for (int d = 0; d < D; d += 4)
            *reinterpret_cast<float4*>(po + d) = make_float4(0.f, 0.f, 0.f, 0.f);
          part_ml[row_id * n_split + it.sp] = make_float2(-INFINITY, 0.f);
        }
        continue;
      }
      const int nt = sp.nt, M = sp.M, n_mt = sp.n_mt;
      const int lim = T_loc - T + tok;  // last visible local key
      const int2* gq = kFused ? groups + (int64_t)it.b * max_groups : nullptr;
      float m_run = -INFINITY, l_run = 0.f;
      for (int j = 0; j < nt; ++j) {
        const uint32_t v = tiles + j;
        if (!*abort_flag && !tc::mbar_wait(&aux.s_full[qt], v & 1)) fail();
        tc::tc_fence_after();
        const int jj = sp.j_lo + j;
        const bool mem = jj < n_mt;
        const int key0 = mem ? jj * kKeys : (jj - n_mt) * kKeys;
        const int n_vis = mem ? min(kKeys, M - key0) : max(0, min(kKeys, lim - key0 + 1));
        uint32_t sv[kKeys];
#pragma unroll
        for (int c = 0; c < kKeys / 32; ++c)
          tc::tmem_ld32(tSP + c * 32, *reinterpret_cast<uint32_t(*)[32]>(sv + c * 32));
        tc::tmem_ld_wait();
        // keys a row may not see read as -inf (also hides whatever S holds
        // there: rows past mem_len, keys past the causal limit)
        bool all8 = true;  // fused memory tile: every row belongs to its document
        if (kFused && mem) {
          // valid rows of each of the tile's 16 groups (0 past the last
          // group), read as the columns reach each group
          for (int gi = 0; gi < kKeys / 8; ++gi) {
            const int grp = key0 / 8 + gi;
            all8 &= grp < M / 8 && gq[grp].y == 8;
          }
          if (!all8) {
            int nvg = 0;
#pragma unroll
            for (int c = 0; c < kKeys; ++c) {
              if ((c & 7) == 0) {
                const int grp = key0 / 8 + (c >> 3);
                nvg = grp < M / 8 ? gq[grp].y : 0;
              }
              if ((c & 7) >= nvg) sv[c] = 0xff800000u;
            }
          }
        } else if (!__all_sync(0xffffffffu, n_vis == kKeys)) {
#pragma unroll
          for (int c = 0; c < kKeys; ++c)
            if (c >= n_vis) sv[c] = 0xff800000u;
        }
        // row maximum: 8 independent chains of 3-input max
        float mx[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) mx[c] = __uint_as_float(sv[c]);
#pragma unroll
        for (int c = 8; c + 16 <= kKeys; c += 16)
#pragma unroll
          for (int u = 0; u < 8; ++u)
            mx[u] = fmax3(mx[u], __uint_as_float(sv[c + u]), __uint_as_float(sv[c + 8 + u]));
        if ((kKeys - 8) % 16)  // the last 8 keys
#pragma unroll
          for (int u = 0; u < 8; ++u) mx[u] = fmaxf(mx[u], __uint_as_float(sv[kKeys - 8 + u]));
        const float mraw = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]),
                                 fmaxf(mx[6], mx[7]));
        const float mt = mraw * qscale;  // qscale > 0 keeps the order
        const bool grow = mt > m_run + kRescaleLog2;
        float alpha = 1.f;
        if (grow) {
          alpha = m_run == -INFINITY ? 0.f : ex2_approx(m_run - mt);
          m_run = mt;
        }
        if (__any_sync(0xffffffffu, grow && alpha != 0.f) && j > 0) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tc::tmem_ld32(tOi + c * 32, o);
            tc::tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(tOi + c * 32, o);
          }
        }
        unsigned char* v_tile = sKV + (v % kStages) * K::STAGE + K::K_BYTES;
        if (!kFused && mem && M - key0 < kKeys) {
          // rows past mem_len in the last memory tile hold whatever the
          // caller's buffer holds there; zero their V so that 0 * V stays 0
          const int vrow = quad * 32 + lane;  // one V row per thread of group 0
          if (qt == 0 && vrow >= M - key0) {
            unsigned char* vp = v_tile + vrow * 128;
#pragma unroll
            for (int kb = 0; kb < K::KB; ++kb)
#pragma unroll
              for (int q = 0; q < 8; ++q)
                *reinterpret_cast<uint4*>(vp + kb * (kKeys * 128) + q * 16) =
                    make_uint4(0, 0, 0, 0);
          }
          tc::fence_proxy_async_smem();
        }
        if (kFused && mem && !all8) {
          // rows of a group past its document's end (and the repeated groups
          // past the query's last one) are other bank rows: their p is 0, and
          // their V is zeroed so that a non-finite bank value cannot turn
          // 0 * V into NaN
          const int vrow = quad * 32 + lane;  // one V row per thread of group 0
          const int grp = key0 / 8 + vrow / 8;
          const int nv = grp < M / 8 ? gq[grp].y : 0;
          if (qt == 0 && (vrow & 7) >= nv) {
            unsigned char* vp = v_tile + vrow * 128;
#pragma unroll
            for (int kb = 0; kb < K::KB; ++kb)
#pragma unroll
              for (int q = 0; q < 8; ++q)
                *reinterpret_cast<uint4*>(vp + kb * (kKeys * 128) + q * 16) =
                    make_uint4(0, 0, 0, 0);
          }
          tc::fence_proxy_async_smem();
        }
        l_run *= alpha;
        const float neg_m = m_run == -INFINITY ? 0.f : -m_run;
        // p = 2^(s * qscale - m_run): the affine step on pairs (f32x2), one
        // ex2 per key, packed to bf16 pairs; the row sum in pairs too
        const unsigned long long sc2 = f2_pack(qscale, qscale), nm2 = f2_pack(neg_m, neg_m);
        unsigned long long ls2[2] = {0ull, 0ull};
#pragma unroll
        for (int c = 0; c < kKeys / 64; ++c) {
          uint32_t w[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int k0 = c * 64 + 2 * e;
            unsigned long long x2 =
                (unsigned long long)sv[k0] | ((unsigned long long)sv[k0 + 1] << 32);
            asm("fma.rn.f32x2 %0, %0, %1, %2;" : "+l"(x2) : "l"(sc2), "l"(nm2));
            const float p0 = ex2_approx(__uint_as_float((uint32_t)x2));
            const float p1 = ex2_approx(__uint_as_float((uint32_t)(x2 >> 32)));
            const unsigned long long p2 = f2_pack(p0, p1);
            asm("add.rn.f32x2 %0, %0, %1;" : "+l"(ls2[e & 1]) : "l"(p2));
            w[e] = pack_bf16(p0, p1);
          }
          tmem_st32(tSP + c * 32, w);  // keys 64c .. 64c+63 -> columns 32c .. 32c+31
        }
        asm("add.rn.f32x2 %0, %0, %1;" : "+l"(ls2[0]) : "l"(ls2[1]));
        const float ls =
            __uint_as_float((uint32_t)ls2[0]) + __uint_as_float((uint32_t)(ls2[0] >> 32));
        l_run += ls;
        tmem_st_wait();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&aux.p_full[qt]);
      }
      // O_i is final once the item's last P V completes; read it out of
      // TMEM, release the columns to the next item's P V, then store
      if (!*abort_flag && !tc::mbar_wait(&aux.o_full[qt], ne & 1)) fail();
      tc::tc_fence_after();
      uint32_t o[D];
#pragma unroll
      for (int c = 0; c < D / 32; ++c)
        tc::tmem_ld32(tOi + c * 32, *reinterpret_cast<uint32_t(*)[32]>(o + c * 32));
      tc::tmem_ld_wait();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&aux.o_empty[qt]);
      tiles += nt;
      ++ne;
      if (!row_ok) continue;
      if (n_split > 1) {
        float* po = part_o + (row_id * n_split + it.sp) * D;
#pragma unroll
        for (int e = 0; e < D; e += 4)
          *reinterpret_cast<float4*>(po + e) =
              make_float4(__uint_as_float(o[e]), __uint_as_float(o[e + 1]),
                          __uint_as_float(o[e + 2]), __uint_as_float(o[e + 3]));
        part_ml[row_id * n_split + it.sp] = make_float2(m_run, l_run);
      } else {
        const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
        __nv_bfloat16* op = out + (((int64_t)it.b * T + tok) * Hq + it.g * G + r % G) * D;
#pragma unroll
        for (int e = 0; e < D; e += 8)
          *reinterpret_cast<uint4*>(op + e) = make_uint4(
              pack_bf16(__uint_as_float(o[e]) * inv, __uint_as_float(o[e + 1]) * inv),
              pack_bf16(__uint_as_float(o[e + 2]) * inv, __uint_as_float(o[e + 3]) * inv),
              pack_bf16(__uint_as_float(o[e + 4]) * inv, __uint_as_float(o[e + 5]) * inv),
              pack_bf16(__uint_as_float(o[e + 6]) * inv, __uint_as_float(o[e + 7]) * inv));
      }
    }
  }

  pdl_trigger();  // this CTA's work is done: the next kernel may be scheduled
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, K::TMEM_COLS);
  }
}

// Global RoPE of the query and the local keys, one launch: CTA p owns local
// position p (query token t sits at local position T_loc - T + t).  The
// kernel is latency-bound at the sizes a step uses, so each thread issues
// the loads of its first 16-byte unit (an element group and its rotate-half
// partner) before the position's (cos, sin) are built in shared memory
// (angle reduced in double, frequencies from the host), then rotates.
//
// Inverse frequencies base^(-2i/D) of a call, computed on the host: the
// kernel keeps only the one double multiply and reduction per (position,
// pair) that an exact angle needs (FP64 is slow on this part, and a double
// pow per thread held the kernel up by microseconds).
struct FreqTab {
  double w[64];
};

template <int D>
__global__ void __launch_bounds__(256)
rope_prep_kernel(int B, int T, int T_loc, int Hq, int H, int64_t pos0,
                 const __grid_constant__ FreqTab freq, const __nv_bfloat16* __restrict__ q,
                 const __nv_bfloat16* __restrict__ k_loc, __nv_bfloat16* __restrict__ q_rot,
                 __nv_bfloat16* __restrict__ k_rot, int* __restrict__ next_item) {
  constexpr int HALF = D / 2;
  constexpr int UPH = HALF / 8;  // 16-byte pair units per head
  // the attention grid that follows may be scheduled now; it waits for this
  // grid's completion before reading what this grid writes.  This grid is
  // itself a programmatic dependent of the work before it (pdl_wait)
  pdl_trigger();
  pdl_wait();
  // the attention grid's item counter: zero once the work before this grid
  // (an earlier attention call that claimed items from it) has completed
  if (blockIdx.x == 0 && threadIdx.x == 0) *next_item = 0;
  __shared__ float2 cs[HALF];
  const int p = blockIdx.x;
  const int tq = p - (T_loc - T);  // query token at this position, if >= 0
  const int nk = B * H * UPH;      // local-key units, then query units
  const int n = nk + (tq >= 0 ? B * Hq * UPH : 0);
  // unit e -> (source, destination offset, pair group)
  auto unit = [&](int e, const __nv_bfloat16*& src, __nv_bfloat16*& dst, int64_t& off, int& u) {
    if (e < nk) {
      u = e % UPH;
      const int h = (e / UPH) % H, b = e / (UPH * H);
      off = (((int64_t)b * T_loc + p) * H + h) * D + u * 8;
      src = k_loc;
      dst = k_rot;
    } else {
      const int f = e - nk;
      u = f % UPH;
      const int h = (f / UPH) % Hq, b = f / (UPH * Hq);
      off = (((int64_t)b * T + tq) * Hq + h) * D + u * 8;
      src = q;
      dst = q_rot;
    }
  };
  auto rotate = [&](const uint4& a, const uint4& bq, __nv_bfloat16* dst, int64_t off, int u) {
    float x1[8], x2[8], y1[8], y2[8];
    Vec16<__nv_bfloat16>::unpack(a, x1);
    Vec16<__nv_bfloat16>::unpack(bq, x2);
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      const float2 c = cs[u * 8 + t];
      y1[t] = x1[t] * c.x - x2[t] * c.y;
      y2[t] = x2[t] * c.x + x1[t] * c.y;
    }
    st16(dst + off, Vec16<__nv_bfloat16>::pack(y1));
    st16(dst + off + HALF, Vec16<__nv_bfloat16>::pack(y2));
  };
  // the first unit's loads are in flight while the table is built
  const int e0 = threadIdx.x;
  const __nv_bfloat16* src0 = nullptr;
  __nv_bfloat16* dst0 = nullptr;
  int64_t off0 = 0;
  int u0 = 0;
  uint4 a0 = make_uint4(0, 0, 0, 0), b0 = a0;
  if (e0 < n) {
    unit(e0, src0, dst0, off0, u0);
    a0 = ldg16(src0 + off0);
    b0 = ldg16(src0 + off0 + HALF);
  }
  for (int i = threadIdx.x; i < HALF; i += blockDim.x) cs[i] = rope_cs(pos0 + p, freq.w[i]);
  __syncthreads();
  if (e0 < n) rotate(a0, b0, dst0, off0, u0);
  for (int e = e0 + blockDim.x; e < n; e += blockDim.x) {
    const __nv_bfloat16* src;
    __nv_bfloat16* dst;
    int64_t off;
    int u;
    unit(e, src, dst, off, u);
    rotate(ldg16(src + off), ldg16(src + off + HALF), dst, off, u);
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

}  // namespace

bool tma_map_sw128_bf16(CUtensorMap* m, const void* ptr, int D, int heads, int64_t rows, int bh,
                        int br) {
  return map3(m, ptr, D, heads, rows, bh, br);
}

bool tma_map_rows_bf16(CUtensorMap* m, const void* ptr, int D, int heads, int64_t rows, int br) {
  auto fn = encode_fn();
  if (!fn || D > 256 || br > 256) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)heads, (cuuint64_t)rows};
  const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)heads * D * 2};
  const cuuint32_t box[3] = {(cuuint32_t)D, 1, (cuuint32_t)br};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

struct TcPlan {
  int n_split;
  size_t q_bytes, k_bytes, po_bytes, ml_bytes, cnt_bytes, total;
};

// Upper bound on key-tile splits: 3, or MSA_ATTN_SPLITS (1..16) from the
// environment, read once.
int max_splits() {
  static const int v = [] {
    const char* e = getenv("MSA_ATTN_SPLITS");
    const int x = e ? atoi(e) : 0;
    return x >= 1 && x <= 16 ? x : 3;
  }();
  return v;
}

// Key-tile splits: enough CTAs to cover the SMs twice, at most max_splits()
// (each split re-reads the query tile and writes an fp32 partial, and the
// combine is one more launch) and at most one per 8 key tiles -- a CTA's
// fixed cost (its query tile, the first tile's latency, the epilogue)
// outweighs a few tiles, so short key ranges are not split.
TcPlan tc_plan(int B, int T, int T_loc, int Hq, int H, int D, int m_cap) {
  TcPlan p{};
  const int G = Hq / H;
  const int TQ = kQT * kRows / G;  // tokens per CTA
  const int64_t base = (int64_t)((T + TQ - 1) / TQ) * H * B;
  const int64_t max_tiles = (m_cap + kKeys - 1) / kKeys + (T_loc + kKeys - 1) / kKeys;
  int64_t ns = (2LL * num_sms() + base - 1) / base;
  ns = std::min<int64_t>(ns, max_splits());
  ns = std::min<int64_t>(ns, max_tiles / 8);
  p.n_split = (int)std::max<int64_t>(ns, 1);
  p.q_bytes = round_up((size_t)B * T * Hq * D * 2, 256);
  p.k_bytes = round_up((size_t)B * T_loc * H * D * 2, 256);
  const size_t rows = (size_t)B * Hq * T;
  p.po_bytes = p.n_split > 1 ? round_up(rows * p.n_split * D * sizeof(float), 256) : 0;
  p.ml_bytes = p.n_split > 1 ? round_up(rows * p.n_split * sizeof(float2), 256) : 0;
  p.cnt_bytes = 256;  // the persistent grid's item counter
  p.total = p.q_bytes + p.k_bytes + p.po_bytes + p.ml_bytes + p.cnt_bytes;
  return p;
}

template <int D>
int launch_tc(int B, int T, int T_loc, int Hq, int H, const void* q, const void* k_mem,
              const void* v_mem, const int32_t* mem_len, int m_cap, const void* k_loc,
              const void* v_loc, int pos0, float rope_base, float qscale, void* out, void* ws,
              cudaStream_t s, const FusedMemory* fm) {
  using K = ACfg<D>;
  const int G = Hq / H;
  if (fm) m_cap = 8 * fm->max_groups;  // memory rows a query can have, for the plan
  const TcPlan p = tc_plan(B, T, T_loc, Hq, H, D, m_cap);
  unsigned char* w = static_cast<unsigned char*>(ws);
  __nv_bfloat16* q_rot = reinterpret_cast<__nv_bfloat16*>(w);
  __nv_bfloat16* k_rot = reinterpret_cast<__nv_bfloat16*>(w + p.q_bytes);
  float* part_o = reinterpret_cast<float*>(w + p.q_bytes + p.k_bytes);
  float2* part_ml = reinterpret_cast<float2*>(w + p.q_bytes + p.k_bytes + p.po_bytes);
  int* next_item = reinterpret_cast<int*>(w + p.q_bytes + p.k_bytes + p.po_bytes + p.ml_bytes);
  FreqTab freq;
  for (int i = 0; i < D / 2; ++i) freq.w[i] = std::pow((double)rope_base, -2.0 * i / D);
  int rc = launch_pdl(rope_prep_kernel<D>, dim3((unsigned)T_loc), dim3(256), 0, s, B, T, T_loc,
                      Hq, H, (int64_t)pos0, freq, static_cast<const __nv_bfloat16*>(q),
                      static_cast<const __nv_bfloat16*>(k_loc), q_rot, k_rot, next_item);
  if (!rc) rc = check_launch();
  if (rc) return rc;

  CUtensorMap tq, tkm, tvm, tkl, tvl;
  const int TQ = kRows / G;  // tokens per Q tile (the TMA box)
  const int64_t mem_rows = std::max<int64_t>((int64_t)B * m_cap, 1);
  const void* km = m_cap > 0 ? k_mem : k_rot;  // any valid address when there is no memory
  const void* vm = m_cap > 0 ? v_mem : v_loc;
  const bool mem_ok =
      fm ? map3(&tkm, fm->k_bar, D, H, fm->n_chunks, 1, 8) &&
               map3(&tvm, fm->v_bar, D, H, fm->n_chunks, 1, 8)
         : map3(&tkm, km, D, H, m_cap > 0 ? mem_rows : (int64_t)B * T_loc, 1, kKeys) &&
               map3(&tvm, vm, D, H, m_cap > 0 ? mem_rows : (int64_t)B * T_loc, 1, kKeys);
  if (!mem_ok || !map3(&tq, q_rot, D, Hq, (int64_t)B * T, G, TQ) ||
      !map3(&tkl, k_rot, D, H, (int64_t)B * T_loc, 1, kKeys) ||
      !map3(&tvl, v_loc, D, H, (int64_t)B * T_loc, 1, kKeys))
    return note_cuda(cudaErrorInvalidValue);
  auto kern = fm ? attn_tc_kernel<D, true> : attn_tc_kernel<D, false>;
  rc = ensure_smem_attr(reinterpret_cast<const void*>(kern), (int)K::SMEM);
  if (rc) return rc;
  const int n_qb = (T + kQT * TQ - 1) / (kQT * TQ);
  const int64_t n_items = (int64_t)n_qb * B * H * p.n_split;
  // items in groups of (batch, KV head) pairs whose key and value rows fit
  // kL2GroupBytes, heaviest first within a group: the CTAs then work on few
  // pairs at a time, and the tiles every query block of a pair re-reads stay
  // in the L2
  const int64_t pair_bytes = (int64_t)(m_cap + T_loc) * D * 2 * 2;
  const int pg =
      (int)std::max<int64_t>(1, std::min<int64_t>((int64_t)B * H, kL2GroupBytes / pair_bytes));
  if (n_items > INT32_MAX / 2) return MSA_ERR_UNSUPPORTED;
  // persistent: one CTA per SM (the shared memory admits one), items claimed
  // at run time
  const dim3 grid((unsigned)std::min<int64_t>(n_items, num_sms()));
  // programmatic dependent launch: the attention grid may be scheduled while
  // the RoPE preparation still runs (its launch latency overlaps it); every
  // thread waits for the preparation's completion (griddepcontrol.wait)
  // before it reads anything, and the preparation itself started only after
  // the work before it in the stream had completed
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = K::SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  rc = note_cuda(cudaLaunchKernelEx(&cfg, kern, tq, tkm, tvm, tkl, tvl, B, T, T_loc, Hq, H, G,
                                    fm ? fm->n_groups : mem_len, m_cap,
                                    fm ? fm->groups : nullptr, fm ? fm->max_groups : 0,
                                    qscale, p.n_split, n_qb, (int)n_items, pg, next_item,
                                    static_cast<__nv_bfloat16*>(out), part_o, part_ml,
                                    device_status_ptr()));
  if (rc) return rc;
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
      (int64_t)B * m_cap > (1LL << 30))
    return false;
  // items: up to 16 splits x H x B x query blocks of kQT * 128 / G tokens
  if ((int64_t)16 * H * B * ((T + kQT * (kRows / G) - 1) / (kQT * (kRows / G))) > INT32_MAX / 2)
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
                         rope_base, qscale, out, ws, s, nullptr);
  return launch_tc<128>(B, T, T_loc, Hq, H, q, k_mem, v_mem, mem_len, m_cap, k_loc, v_loc, pos0,
                        rope_base, qscale, out, ws, s, nullptr);
}

size_t attn_tc_fused_workspace_size(int B, int T, int T_loc, int Hq, int H, int D,
                                    int max_groups) {
  return tc_plan(B, T, T_loc, Hq, H, D, 8 * max_groups).total;
}

int attn_tc_launch_fused(int B, int T, int T_loc, int Hq, int H, int D, const void* q,
                         const FusedMemory& fm, const void* k_loc, const void* v_loc, int pos0,
                         float rope_base, float qscale, void* out, void* ws, cudaStream_t s) {
  if (!aligned16(q) || !aligned16(k_loc) || !aligned16(v_loc) || !aligned16(out) ||
      !aligned16(fm.k_bar) || !aligned16(fm.v_bar))
    return MSA_ERR_INVALID_ARG;
  if (D == 64)
    return launch_tc<64>(B, T, T_loc, Hq, H, q, nullptr, nullptr, nullptr, 0, k_loc, v_loc,
                         pos0, rope_base, qscale, out, ws, s, &fm);
  return launch_tc<128>(B, T, T_loc, Hq, H, q, nullptr, nullptr, nullptr, 0, k_loc, v_loc, pos0,
                        rope_base, qscale, out, ws, s, &fm);
}

}  // namespace msa
