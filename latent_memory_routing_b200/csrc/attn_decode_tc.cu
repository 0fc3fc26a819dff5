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
// instructions left per key hide under the stream.  A persistent grid of at
// most one CTA of 15 warps per SM takes work items -- a chunk of consecutive
// key tiles of one (batch element, KV head), serving the G query heads of
// the KV head padded to N = 16 MMA columns -- from a global counter as it
// goes (a CTA that runs faster takes more, so the CTAs end together), with
// one continuous pipeline across items, so the stream never drains between
// them:
//   * warp 0 TMA-loads 128-key K and V tiles (128B-swizzled, 64-dim blocks)
//     into 3-slot K and V rings, one lane each -- the K lane also takes the
//     next chunk and publishes it to the other roles -- per item, memory tiles
//     first, then local tiles, so no tile mixes the two; a K slot is
//     released when S has read it, a V slot when P V has, so the K stream
//     runs ahead;
//   * warps 2, 3, 8..13 (rotators) apply RoPE to local K tiles in shared
//     memory in the relative form <R(p_q) q, R(p_k) k> = <R(Delta) q,
//     R(delta) k>: a key's rotation by its offset delta in the tile, and
//     the query, rotated per tile by the tile's distance Delta to it (one
//     complex step per tile from an anchor the host computed exactly), is
//     written as the MMA's B operand; memory keys are not rotated and meet
//     R(p_q) q;
//   * warp 1 issues S^T = K Q^T (M = 128 keys, N = 16, K = 128) into one of
//     two TMEM buffers as soon as a K tile is rotated, and the last warp
//     issues O^T += V^T P^T (M = 128 dims, N = 16, K = 128 keys; V read
//     MN-major) into the O^T TMEM columns as soon as P and the V tile are
//     there -- two issuers, so that S never queues behind a P V that waits
//     for its V tile (the V stream, whose slots are held longest, sets the
//     pace);
//   * warps 4..7 (softmax, one thread per TMEM lane: a key row of S^T, a dim
//     row of O^T) turn S into P (base-2 exponent domain, the scale folded
//     into Q) against a per-head reference maximum that moves only when a
//     score exceeds it by more than 2^8 -- then O^T is rescaled in TMEM --,
//     keep per-thread partial row sums (reduced once at the end), and write
//     P^T (bf16) as the B operand of P V (a masked memory row -- past
//     mem_len, or past its document's end in the fused form -- also has its
//     V row zeroed in shared memory); at an item's last tile they reduce
//     the row sums and write the item's output.
// The query buffers are double-buffered by item and by tile.  The chunks of
// one (batch element, KV head) write (max, sum, O) partials, and the last of
// them to finish merges them into the output (an arrival counter), so no
// second launch combines them; a lone chunk writes the output directly.  The
// RoPE constants come from the host (no double-precision arithmetic on the
// device), so nothing precedes the kernel but the reset of its counters.
// Every wait is bounded; after a timeout every role walks its loop without
// waiting.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdlib>

#include "attn_tc.cuh"
#include "msa_common.cuh"
#include "tc_ptx.cuh"

namespace msa {
namespace {

constexpr int kTK = 128;                   // keys per tile (M of S^T)
constexpr int kNH = 16;                    // MMA columns: G <= 16 heads, padded
constexpr int kDim = 128;                  // head dim
// K and V rings of 128-key tiles: a K slot is held from its load to S, a V
// slot from its load to P V (after S and the softmax), so the V ring is the
// deeper one
#ifndef MSA_DTC_KST
#define MSA_DTC_KST 3
#endif
#ifndef MSA_DTC_VST
#define MSA_DTC_VST 3
#endif
constexpr int kKSt = MSA_DTC_KST;
constexpr int kVSt = MSA_DTC_VST;

constexpr int kRotWarps = 8;
constexpr int kSoftWarps = 4;
constexpr int kPvWarp = 2 + kRotWarps + kSoftWarps;  // the P V issuer, last warp
constexpr int kTThreads = 32 * (kPvWarp + 1);
constexpr int kBlk = kTK * 128;            // one 64-dim block of a K or V tile: 16 KB
constexpr int kTileBytes = 2 * kBlk;       // K or V tile: 32 KB
constexpr int kQBytes = kNH * kDim * 2;    // Q [16][128] bf16: two 2 KB blocks
constexpr int kPBytes = kNH * kTK * 2;     // P^T [16][128] bf16: two 2 KB blocks
constexpr int kSmBar = 1;                  // named barrier of the softmax warps
constexpr float kRescaleLog2 = 8.f;
constexpr uint32_t kIdescS = tc::idesc_bf16_f32(kTK, kNH);
constexpr uint32_t kIdescO = tc::idesc_bf16_f32(kDim, kNH) | (1u << 15);  // A MN-major
constexpr uint32_t kTmemCols = 64;         // S buffers: 0..31, O^T: 32..47

struct DTS {  // dynamic shared memory, offsets from a 1024-byte aligned base
  static constexpr size_t RING = 0;
  static constexpr size_t VRING = RING + (size_t)kKSt * kTileBytes;
  static constexpr size_t QMEM = VRING + (size_t)kVSt * kTileBytes;  // [2] by item
  static constexpr size_t QT = QMEM + 2 * kQBytes;   // [2] by tile
  static constexpr size_t P = QT + 2 * kQBytes;      // [2] by tile
  static constexpr size_t QRAW = P + 2 * kPBytes;    // [2][16][128] bf16 raw query, by item
  static constexpr size_t RED = QRAW + 2 * (size_t)kNH * kDim * 2;  // [4][16] f32
  static constexpr size_t FLAGS = RED + 4 * kNH * 4;            // [2][4] int + 4 int
  static constexpr size_t ALLOC = FLAGS + 3 * 4 * 4 + 1024;
  static_assert(QMEM % 1024 == 0 && QT % 1024 == 0 && P % 1024 == 0, "swizzle atoms");
  static_assert(ALLOC <= 227 * 1024, "shared memory per CTA");
};

// Ring of chunk ids published by the K producer: read by the V producer,
// the two MMA issuers (one lane each), the softmax warps and the rotator
// warps (one arrival per warp).
constexpr int kSched = 4;
constexpr int kSchedReaders = 3 + kSoftWarps + kRotWarps;

struct DTAux {
  // K and V tiles of a stage arrive and leave separately: a K slot is free
  // once S has read it, a V slot once P V has
  uint64_t kfull[kKSt], vfull[kVSt], kready[kKSt], kfree[kKSt], vfree[kVSt];
  uint64_t sfull[2], sfree[2], pfull[2], pvdone[2], odone;
  uint64_t sched_full[kSched], sched_empty[kSched];
  int sched_id[kSched];
  uint32_t tmem_base;
  int abort_flag;
};

// RoPE constants of a call, computed on the host in double and rounded
// once: the kernel does no double-precision arithmetic (FP64 is slow on this
// part, and a handful of double operations per thread held up the first
// tiles by microseconds).  For pair i (of kDim / 2):
//   w[i]      inverse frequency base^(-2i/D);
//   qpos[i]   R(p_q w_i), the query's own position p_q = pos0 + T_loc - 1;
//   qdelta[i] R((T_loc - 1) w_i), the distance from local key 0 to the query;
//   qstep[i]  R(kTK w_i), one key tile.
struct RopeTab {
  float w[kDim / 2];
  float2 qpos[kDim / 2], qdelta[kDim / 2], qstep[kDim / 2];
};

// Complex product a * conj(b): rotation by angle(a) - angle(b).
__device__ __forceinline__ float2 cmul_conj(float2 a, float2 b) {
  return make_float2(a.x * b.x + a.y * b.y, a.y * b.x - a.x * b.y);
}
__device__ __forceinline__ float2 cmul(float2 a, float2 b) {
  return make_float2(a.x * b.x - a.y * b.y, a.x * b.y + a.y * b.x);
}

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

// One work item: a chunk of the key tiles of one (batch element, KV head).
// Chunks are handed out at run time: the K producer lane takes the next
// chunk id from a global counter (atomicAdd) when it has issued the last
// loads of its current chunk and publishes it in a small shared-memory ring;
// every other role reads the ring in the same order, so all roles walk the
// same sequence -- chunks with no tiles skipped -- through their own cursor.
// A CTA that runs ahead takes more chunks, so the CTAs end together.
struct Cur {
  int su;                // ring entries read (or, for the K producer, published)
  int k, j, nt;          // ordinal of the chunk among this CTA's non-empty ones, tile, tiles
  int item, b, g, sp, n_eff, M, n_mt, j_lo;
};

// kFused: the memory rows come straight from the pooled bank -- per query
// a list of 8-row groups (first bank row, rows that belong to the document)
// in rank order -- instead of a gathered [B][m_cap] buffer; tm_km / tm_vm
// then map the bank with 8-row boxes (one 128B-swizzle atom each), and a
// memory tile is 16 groups.  Rows past a document's end within its last
// group are other bank rows: masked out, and their V zeroed in shared memory
// by the softmax (as the rows past mem_len of a gathered memory tile).
//
// Chunk ids: the first n_whole ids are whole items (item = id; item =
// b * H + g).  Whole items fill complete rounds of the grid; the remaining
// n_tail items, which would leave most CTAs idle in a last partial round,
// are cut into chunks: id = n_whole + sp * n_tail + t is chunk sp of item
// n_whole + t, and an item of nt key tiles is cut into n_eff = min(n_ch, nt)
// chunks of consecutive tiles (chunks sp >= n_eff hold none).  A cut item's
// chunks write (max, sum, O) partials; the last of them to finish (an
// arrival counter per cut item) merges them and writes the output, so no
// second launch combines them.  counters[0] (chunk counter) and
// counters[1 + t] (arrivals) are zero at launch.
template <int G, bool kFused>
__global__ void __launch_bounds__(kTThreads, 1)
attn_decode_tc_kernel(const __grid_constant__ CUtensorMap tm_km,
                      const __grid_constant__ CUtensorMap tm_vm,
                      const __grid_constant__ CUtensorMap tm_kl,
                      const __grid_constant__ CUtensorMap tm_vl, int T_loc, int Hq, int H,
                      int n_whole, int n_tail, int n_ch, const __nv_bfloat16* __restrict__ q,
                      const int32_t* __restrict__ mem_len, int m_cap,
                      const int2* __restrict__ groups, int max_groups,
                      const __grid_constant__ RopeTab rope, float qscale,
                      int* __restrict__ counters,
                      __nv_bfloat16* __restrict__ out, float* __restrict__ part_o,
                      float2* __restrict__ part_ml, int* __restrict__ status) {
  static_assert(G >= 1 && G <= kNH, "heads per KV head");
  constexpr int HALF = kDim / 2;
  extern __shared__ __align__(1024) unsigned char dsm[];
  __shared__ DTAux aux;
  unsigned char* sm = tc::smem_align<1024>(dsm);
  unsigned char* ring = sm + DTS::RING;    // K ring
  unsigned char* vring = sm + DTS::VRING;  // V ring
  unsigned char* qmem = sm + DTS::QMEM;  // [2] by chunk
  unsigned char* qt = sm + DTS::QT;      // [2] by tile
  unsigned char* pbuf = sm + DTS::P;     // [2] by tile
  __nv_bfloat16* qraw = reinterpret_cast<__nv_bfloat16*>(sm + DTS::QRAW);  // [2][16][128]
  float* red = reinterpret_cast<float*>(sm + DTS::RED);
  int* flags = reinterpret_cast<int*>(sm + DTS::FLAGS);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n_chunks = n_whole + n_tail * n_ch;
  const int n_lt = (T_loc + kTK - 1) / kTK;

  auto load_chunk = [&](Cur& c, int id) {
    if (id < n_whole) {
      c.sp = 0;
      c.item = id;
    } else {
      c.sp = (id - n_whole) / n_tail;
      c.item = n_whole + (id - n_whole) % n_tail;
    }
    c.b = c.item / H;
    c.g = c.item % H;
    // fused: mem_len holds the query's group count; its memory is 8 rows a group
    c.M = kFused ? 8 * min(max(mem_len[c.b], 0), max_groups) : min(max(mem_len[c.b], 0), m_cap);
    c.n_mt = (c.M + kTK - 1) / kTK;
    const int n_all = c.n_mt + n_lt;
    c.n_eff = c.item < n_whole ? 1 : min(n_ch, n_all);
    if (c.sp >= c.n_eff) {
      c.nt = 0;
      return;
    }
    c.j_lo = (int)((int64_t)c.sp * n_all / c.n_eff);
    c.nt = (int)((int64_t)(c.sp + 1) * n_all / c.n_eff) - c.j_lo;
  };
  volatile int* abort_flag = &aux.abort_flag;
  auto wait_or_abort = [&](uint64_t* bar, uint32_t parity) {
    if (*abort_flag) return;
    if (!tc::mbar_wait(bar, parity)) {
      record_error(status, MSA_ERR_TIMEOUT);
      *abort_flag = 1;
    }
  };
  // K producer: take the next chunk from the counter and publish it.  The
  // counter is read early (`ahead`, taken as the current chunk's last tile
  // is issued) so that its round trip overlaps that tile's load.
  int ahead = -1;
  auto grab = [&](Cur& c) -> bool {
    for (;;) {
      const int slot = c.su % kSched;
      wait_or_abort(&aux.sched_empty[slot], ((c.su / kSched) & 1) ^ 1);
      int id = -1;
      if (!*abort_flag) {
        const int t = ahead >= 0 ? ahead : atomicAdd(counters, 1);
        ahead = -1;
        id = t < n_chunks ? t : -1;
      }
      aux.sched_id[slot] = id;
      tc::mbar_arrive(&aux.sched_full[slot]);  // release: the id is visible to the waiters
      ++c.su;
      if (id < 0) return false;
      load_chunk(c, id);
      if (c.nt > 0) {
        c.j = 0;
        return true;
      }
    }
  };
  // every other role: read the next published chunk (`whole_warp`: all 32
  // lanes read, lane 0 arrives for the warp)
  auto fetch = [&](Cur& c, bool whole_warp) -> bool {
    for (;;) {
      const int slot = c.su % kSched;
      wait_or_abort(&aux.sched_full[slot], (c.su / kSched) & 1);
      const int id = *abort_flag ? -1 : aux.sched_id[slot];
      if (whole_warp) __syncwarp();
      if (!whole_warp || lane == 0) tc::mbar_arrive(&aux.sched_empty[slot]);
      ++c.su;
      if (id < 0) return false;
      load_chunk(c, id);
      if (c.nt > 0) {
        c.j = 0;
        return true;
      }
    }
  };
  auto first = [&](Cur& c, int role) -> bool {
    c.su = 0;
    c.k = 0;
    return role == 0 ? grab(c) : fetch(c, role == 2);
  };
  auto next = [&](Cur& c, int role) -> bool {
    if (++c.j < c.nt) return true;
    ++c.k;
    return role == 0 ? grab(c) : fetch(c, role == 2);
  };
  auto tile_mem = [&](const Cur& c) { return c.j_lo + c.j < c.n_mt; };
  auto tile_key0 = [&](const Cur& c) {
    const int jj = c.j_lo + c.j;
    return jj < c.n_mt ? jj * kTK : (jj - c.n_mt) * kTK;
  };
  auto tile_valid = [&](const Cur& c) {
    const int jj = c.j_lo + c.j;
    return jj < c.n_mt ? min(kTK, c.M - jj * kTK) : min(kTK, T_loc - (jj - c.n_mt) * kTK);
  };

  if (tid == 0) {
    for (int i = 0; i < kKSt; ++i) {
      tc::mbar_init(&aux.kfull[i], 1);
      tc::mbar_init(&aux.kready[i], kRotWarps);
      tc::mbar_init(&aux.kfree[i], 1);
    }
    for (int i = 0; i < kVSt; ++i) {
      tc::mbar_init(&aux.vfull[i], 1);
      tc::mbar_init(&aux.vfree[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&aux.sfull[i], 1);
      tc::mbar_init(&aux.sfree[i], kSoftWarps);
      tc::mbar_init(&aux.pfull[i], kSoftWarps);
    }
    tc::mbar_init(&aux.pvdone[0], 1);
    tc::mbar_init(&aux.pvdone[1], 1);
    tc::mbar_init(&aux.odone, 1);
    for (int i = 0; i < kSched; ++i) {
      tc::mbar_init(&aux.sched_full[i], 1);
      tc::mbar_init(&aux.sched_empty[i], kSchedReaders);
    }
    aux.abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(&aux.tmem_base, kTmemCols);
    tc::tmem_relinquish();
  }
  // all query and P^T buffers start at zero (rows >= G stay zero)
  for (int e = tid; e < (4 * kQBytes + 2 * kPBytes) / 16; e += kTThreads)
    reinterpret_cast<uint4*>(qmem)[e] = make_uint4(0, 0, 0, 0);
  tc::fence_proxy_async_smem();
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = aux.tmem_base;

  if (warp == 0) {
    // ----------------------------------------------------------- producers
    // lane 0 streams the K tiles (and takes the chunks), lane 1 the V tiles,
    // each gated by its own slot releases, so K loads run ahead of the V
    // slots P V still holds
    if (lane < 2) {
      const bool isv = lane == 1;
      const int role = isv ? 1 : 0;
      uint64_t* fullb = isv ? aux.vfull : aux.kfull;
      const int nst = isv ? kVSt : kKSt;
      uint64_t* freeb = isv ? aux.vfree : aux.kfree;
      Cur c;
      int u = 0;
      for (bool ok = first(c, role); ok; ok = next(c, role), ++u) {
        const int st = u % nst;
        if (!isv && c.j == c.nt - 1) ahead = atomicAdd(counters, 1);  // the next chunk
        const bool mem = tile_mem(c);
        // fused memory tile: its 16 groups' first bank rows, all read before
        // the slot wait (one round trip, overlapping it; the TMA issue below
        // is ordered after every memory access, so a read between two issues
        // would cost a round trip per group); past the query's last group,
        // the last one again (masked, V zeroed) so every row of the tile is
        // written
        int src[kTK / 8];
        if (kFused && mem) {
          const int ng = c.M / 8, g0 = tile_key0(c) / 8;
          const int2* gq = groups + (int64_t)c.b * max_groups;
#pragma unroll
          for (int gi = 0; gi < kTK / 8; ++gi) src[gi] = __ldg(&gq[min(g0 + gi, ng - 1)].x);
        }
        wait_or_abort(&freeb[st], ((u / nst) & 1) ^ 1);
        if (*abort_flag) break;
        unsigned char* d = (isv ? vring : ring) + (size_t)st * kTileBytes;
        const CUtensorMap* m = mem ? (isv ? &tm_vm : &tm_km) : (isv ? &tm_vl : &tm_kl);
        tc::mbar_arrive_expect_tx(&fullb[st], kTileBytes);
        if (kFused && mem) {
          // 16 groups of 8 bank rows
#pragma unroll
          for (int gi = 0; gi < kTK / 8; ++gi) {
            tc::tma_load_3d(d + gi * 1024, m, &fullb[st], 0, c.g, src[gi]);
            tc::tma_load_3d(d + kBlk + gi * 1024, m, &fullb[st], 64, c.g, src[gi]);
          }
        } else {
          const int row0 = (mem ? c.b * m_cap : c.b * T_loc) + tile_key0(c);
          tc::tma_load_3d(d, m, &fullb[st], 0, c.g, row0);
          tc::tma_load_3d(d + kBlk, m, &fullb[st], 64, c.g, row0);
        }

      }
      for (int v = u > nst ? u - nst : 0; v < u; ++v)
        tc::mbar_wait(&fullb[v % nst], (v / nst) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- S MMA
    // S(u) as soon as its K tile is rotated (kready) and its TMEM buffer
    // u&1 has been read by the softmax of tile u-2 (sfree of u-2, which the
    // softmax signals as soon as S is in its registers): the P V stream,
    // issued by its own warp, does not hold it back
    if (lane == 0) {
      Cur cs;
      int us = 0;
      for (bool hs = first(cs, 1); hs; hs = next(cs, 1), ++us) {
        const int st = us % kKSt;
        wait_or_abort(&aux.kready[st], (us / kKSt) & 1);
        if (us >= 2) wait_or_abort(&aux.sfree[us & 1], ((us - 2) >> 1) & 1);
        tc::tc_fence_after();
        const uint64_t ad = tc::sdesc_kmajor_sw128(tc::smem_u32(ring + (size_t)st * kTileBytes));
        const uint64_t bd = tc::sdesc_kmajor_sw128(
            tc::smem_u32(tile_mem(cs) ? qmem + (cs.k & 1) * kQBytes : qt + (us & 1) * kQBytes));
#pragma unroll
        for (int kk = 0; kk < kDim / 16; ++kk) {
          const uint32_t koff = (kk & 3) * 32;
          tc::mma_bf16_ss(tmem + (us & 1) * kNH, tc::desc_add(ad, (kk >> 2) * kBlk + koff),
                          tc::desc_add(bd, (kk >> 2) * (kNH * 128) + koff), kIdescS,
                          kk > 0 ? 1u : 0u);
        }
        tc::mma_commit(&aux.sfull[us & 1]);
        tc::mma_commit(&aux.kfree[st]);  // S has read the K slot
      }
    }
  } else if (warp == kPvWarp) {
    // ----------------------------------------------------------- P V MMA
    // P V(u) as soon as P(u) is written and V(u) has landed
    if (lane == 0) {
      Cur cp;
      int up = 0;
      for (bool hp = first(cp, 1); hp; hp = next(cp, 1), ++up) {
        const int st = up % kVSt;
        wait_or_abort(&aux.pfull[up & 1], (up >> 1) & 1);
        wait_or_abort(&aux.vfull[st], (up / kVSt) & 1);
        tc::tc_fence_after();
        const uint64_t vd =
            tc::sdesc_mnmajor_sw128(tc::smem_u32(vring + (size_t)st * kTileBytes), kBlk);
        const uint64_t pd = tc::sdesc_kmajor_sw128(tc::smem_u32(pbuf + (up & 1) * kPBytes));
        const bool first_tile = cp.j == 0, last_tile = cp.j == cp.nt - 1;
#pragma unroll
        for (int kk = 0; kk < kTK / 16; ++kk)
          tc::mma_bf16_ss(tmem + 2 * kNH, tc::desc_add(vd, kk * 16 * 128),
                          tc::desc_add(pd, (kk >> 2) * (kNH * 128) + (kk & 3) * 32), kIdescO,
                          (!first_tile || kk > 0) ? 1u : 0u);
        tc::mma_commit(&aux.vfree[st]);        // P V has read the V slot
        tc::mma_commit(&aux.pvdone[up & 1]);   // ... and the P buffer up&1
        if (last_tile) tc::mma_commit(&aux.odone);  // this chunk's O^T is final
      }
    }
  } else if (warp >= 4 && warp < 4 + kSoftWarps) {
    // ------------------------------------------------------------- softmax
    const int w4 = warp - 4;            // TMEM lane quarter
    const int r = w4 * 32 + lane;       // key row of S^T, dim row of O^T
    const uint32_t lane_addr = (uint32_t)(w4 * 32) << 16;
    float m_ref[G], l_part[G];
    Cur c;
    int u = 0;
    for (bool ok = first(c, 2); ok; ok = next(c, 2), ++u) {
      if (c.j == 0) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
          m_ref[h] = -INFINITY;
          l_part[h] = 0.f;
        }
      }
      wait_or_abort(&aux.sfull[u & 1], (u >> 1) & 1);
      tc::tc_fence_after();
      uint32_t sv[16];
      tc::tmem_ld16(tmem + lane_addr + (u & 1) * kNH, sv);
      tc::tmem_ld_wait();
      // S(u) is in registers: its TMEM buffer may take S(u + 2)
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&aux.sfree[u & 1]);
      bool valid = r < tile_valid(c);
      if (kFused && tile_mem(c)) {  // its group holds the row, and the row its document's
        const int grp = (tile_key0(c) + r) / 8;
        valid = grp < c.M / 8 && (r & 7) < groups[(int64_t)c.b * max_groups + grp].y;
      }
      if (!valid && tile_mem(c)) {
        // this memory row lies past mem_len (whatever the caller's buffer
        // holds there) or past its document's end (another document's bank
        // row): zero its V once it has landed, so that 0 * V stays 0 in P V.
        // P V waits for this thread's pfull arrival below, so V(u + kVSt)
        // cannot land in the slot before P V(u) has released it; and P V of
        // tile u-3, awaited for tile u-1, means every earlier V has landed:
        // the parity of tile u names this tile.
        const int st = u % kVSt;
        wait_or_abort(&aux.vfull[st], (u / kVSt) & 1);
        unsigned char* vt = vring + (size_t)st * kTileBytes;
#pragma unroll
        for (int cc = 0; cc < 16; ++cc)
          *reinterpret_cast<uint4*>(vt + (cc >> 3) * kBlk + r * 128 + ((cc & 7) << 4)) =
              make_uint4(0, 0, 0, 0);
      }
      float s[G];
      bool need = false;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        s[h] = valid ? __uint_as_float(sv[h]) : -INFINITY;
        need |= s[h] > m_ref[h] + kRescaleLog2;
      }
      const int any_w = __any_sync(0xffffffffu, need);
      int* fl = flags + (u & 1) * 4;
      if (lane == 0) fl[w4] = any_w;
      soft_bar();
      if (fl[0] | fl[1] | fl[2] | fl[3]) {  // uniform: new reference maxima
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
          const float mt =
              fmaxf(fmaxf(red[h], red[kNH + h]), fmaxf(red[2 * kNH + h], red[3 * kNH + h]));
          alpha[h] = 1.f;
          if (mt > m_ref[h] + kRescaleLog2) {
            alpha[h] = m_ref[h] == -INFINITY ? 0.f : ex2a(m_ref[h] - mt);
            m_ref[h] = mt;
            rescale = true;
          }
          l_part[h] *= alpha[h];
        }
        if (rescale && c.j > 0) {
          // O^T holds P V of this chunk's earlier tiles: wait for the last
          // one (tile u-1), then scale each head's column in TMEM
          wait_or_abort(&aux.pvdone[(u - 1) & 1], ((u - 1) >> 1) & 1);
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
      // P^T column of this key into buffer u&1, once its previous reader,
      // P V of tile u-2, is done
      if (u >= 2) wait_or_abort(&aux.pvdone[u & 1], ((u - 2) >> 1) & 1);
      unsigned char* pb = pbuf + (u & 1) * kPBytes;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float p = (valid && m_ref[h] != -INFINITY) ? ex2a(s[h] - m_ref[h]) : 0.f;
        l_part[h] += p;
        *reinterpret_cast<__nv_bfloat16*>(pb + sw128_off(h, r, kNH)) = __float2bfloat16(p);
      }
      tc::fence_proxy_async_smem();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&aux.pfull[u & 1]);
      if (c.j == c.nt - 1) {
        // the chunk's last tile: once its P V is done, reduce the row sums
        // over the 128 key lanes and write this chunk's O (dim r per thread)
        wait_or_abort(&aux.odone, c.k & 1);
        tc::tc_fence_after();
        soft_bar();  // every thread is past its reads of red
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
        tc::tc_fence_before();  // the next chunk's first P V overwrites O^T
        const int64_t row0 = (int64_t)c.item * G;  // = b * Hq + g * G (T == 1)
        if (c.n_eff == 1) {
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const float l = red[h] + red[kNH + h] + red[2 * kNH + h] + red[3 * kNH + h];
            const float o = __uint_as_float(ov[h]);
            out[(row0 + h) * kDim + r] = __float2bfloat16(l > 0.f ? o / l : 0.f);
          }
        } else {
          const int tail = c.item - n_whole;  // cut items only
          const int64_t pidx = (int64_t)tail * n_ch + c.sp;
#pragma unroll
          for (int h = 0; h < G; ++h) {
            part_o[(pidx * G + h) * kDim + r] = __uint_as_float(ov[h]);
            if (r == 0) {
              const float l = red[h] + red[kNH + h] + red[2 * kNH + h] + red[3 * kNH + h];
              part_ml[pidx * G + h] = make_float2(m_ref[h], l);
            }
          }
          // publish the partial, then count this chunk's arrival; the last
          // of the item's n_eff chunks merges them.  The group barrier orders
          // every thread's partial before the counting thread's device-scope
          // fence and atomic (the fence is cumulative), and the merging
          // side's fence orders the count before its reads.
          soft_bar();
          if (r == 0) {
            __threadfence();
            flags[8] = atomicAdd(counters + 1 + tail, 1) == c.n_eff - 1;
          }
          soft_bar();
          if (flags[8]) {
            __threadfence();
            const int64_t p0 = (int64_t)tail * n_ch;
            // online merge, kMB chunks at a time with every load of a batch
            // issued before its arithmetic (G * kMB <= 16 loads of each kind
            // in flight): the running maximum rescales what came before
            constexpr int kMB = G >= 16 ? 1 : (G >= 8 ? 2 : 4);
            float mx[G], l[G], acc[G];
#pragma unroll
            for (int h = 0; h < G; ++h) {
              mx[h] = -INFINITY;
              l[h] = 0.f;
              acc[h] = 0.f;
            }
            for (int s0 = 0; s0 < c.n_eff; s0 += kMB) {
              float2 ml[kMB][G];
              float o[kMB][G];
#pragma unroll
              for (int i = 0; i < kMB; ++i)
#pragma unroll
                for (int h = 0; h < G; ++h) {
                  const bool live = s0 + i < c.n_eff;
                  const int64_t pi = (p0 + s0 + i) * G + h;
                  ml[i][h] = live ? __ldcg(&part_ml[pi]) : make_float2(-INFINITY, 0.f);
                  o[i][h] = live ? __ldcg(&part_o[pi * kDim + r]) : 0.f;
                }
#pragma unroll
              for (int i = 0; i < kMB; ++i)
#pragma unroll
                for (int h = 0; h < G; ++h) {
                  if (ml[i][h].x == -INFINITY) continue;
                  const float mn = fmaxf(mx[h], ml[i][h].x);
                  const float a = exp2f(mx[h] - mn), wgt = exp2f(ml[i][h].x - mn);
                  l[h] = l[h] * a + wgt * ml[i][h].y;
                  acc[h] = acc[h] * a + wgt * o[i][h];
                  mx[h] = mn;
                }
            }
#pragma unroll
            for (int h = 0; h < G; ++h)
              out[(row0 + h) * kDim + r] = __float2bfloat16(l[h] > 0.f ? acc[h] / l[h] : 0.f);
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ rotators
    const int rt = (warp < 4 ? warp - 2 : warp - 6) * 32 + lane;  // 0 .. 255
    const int ch = rt & 7, r0 = rt >> 3;  // 16-byte chunk, first of four rows
    // RoPE in the relative form <R(p_q) q, R(p_k) k> = <R(Delta) q, R(delta) k>
    // for a local tile: a key's rotation by its offset delta in the tile and
    // the query's by the tile's distance Delta to it.  Thread rt rotates rows
    // r0 + 32 qq (qq = 0..3), pairs i = 8 ch + e (e = 0..7): their
    // R(delta w_i) come from fp32 angles delta * w_i < 128 rad (error
    // <= ~1.5e-5 rad, two orders below the bf16 rounding of the rotated key).
    float2 cs[4][8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float wi = rope.w[8 * ch + e];
#pragma unroll
      for (int qq = 0; qq < 4; ++qq) {
        float sn, cn;
        sincosf((float)(r0 + 32 * qq) * wi, &sn, &cn);
        cs[qq][e] = make_float2(cn, sn);
      }
    }
    const int i_q = rt % HALF;  // query pair this thread rotates (every chunk)
    const float2 qstep = rope.qstep[i_q];
    const float2 qpos = rope.qpos[i_q];  // R(p_q) for memory tiles
    float2 qcs = make_float2(1.f, 0.f);
    bool anchored = false;
    Cur c;
    int u = 0;
    for (bool ok = first(c, 2); ok; ok = next(c, 2), ++u) {
      const int st = u % kKSt;
      wait_or_abort(&aux.kfull[st], (u / kKSt) & 1);
      unsigned char* kt = ring + (size_t)st * kTileBytes;
      __nv_bfloat16* qr = qraw + (c.k & 1) * kNH * kDim;
      if (c.j == 0) {
        // a new chunk: its raw query and R(p_q) q go to buffers k&1, whose
        // last readers (S of chunk k-2, at or before tile u-1) must be done
        if (u >= 1) wait_or_abort(&aux.sfull[(u - 1) & 1], ((u - 1) >> 1) & 1);
        for (int e = rt; e < G * kDim; e += 32 * kRotWarps)
          qr[e] = q[((int64_t)c.b * Hq + c.g * G) * kDim + e];
        asm volatile("bar.sync %0, %1;" ::"n"(kSmBar + 1), "n"(32 * kRotWarps) : "memory");
        if (c.n_mt > c.j_lo) {
          unsigned char* qm = qmem + (c.k & 1) * kQBytes;
          for (int e = rt; e < G * HALF; e += 32 * kRotWarps) {
            const int h = e / HALF;
            const float x1 = __bfloat162float(qr[h * kDim + i_q]) * qscale;
            const float x2 = __bfloat162float(qr[h * kDim + i_q + HALF]) * qscale;
            *reinterpret_cast<__nv_bfloat16*>(qm + sw128_off(h, i_q, kNH)) =
                __float2bfloat16(x1 * qpos.x - x2 * qpos.y);
            *reinterpret_cast<__nv_bfloat16*>(qm + sw128_off(h, i_q + HALF, kNH)) =
                __float2bfloat16(x2 * qpos.x + x1 * qpos.y);
          }
        }
        anchored = false;
      }
      if (!tile_mem(c)) {
        // R(Delta) q into buffer u&1, whose last reader S(u-2) must be done
        if (u >= 2) wait_or_abort(&aux.sfull[u & 1], ((u - 2) >> 1) & 1);
        if (!anchored) {
          // Delta = (T_loc - 1) - kTK t for the chunk's first local tile t:
          // R((T_loc - 1) w) R(kTK w)^(-t), the power by repeated squaring
          int t = tile_key0(c) / kTK;
          float2 sq = qstep;
          qcs = rope.qdelta[i_q];
          while (t) {
            if (t & 1) qcs = cmul_conj(qcs, sq);
            sq = cmul(sq, sq);
            t >>= 1;
          }
          anchored = true;
        } else {  // Delta fell by kTK: multiply by e^{-i kTK w}
          qcs = cmul_conj(qcs, qstep);
        }
        unsigned char* qb = qt + (u & 1) * kQBytes;
        for (int e = rt; e < G * HALF; e += 32 * kRotWarps) {
          const int h = e / HALF;
          const float x1 = __bfloat162float(qr[h * kDim + i_q]) * qscale;
          const float x2 = __bfloat162float(qr[h * kDim + i_q + HALF]) * qscale;
          *reinterpret_cast<__nv_bfloat16*>(qb + sw128_off(h, i_q, kNH)) =
              __float2bfloat16(x1 * qcs.x - x2 * qcs.y);
          *reinterpret_cast<__nv_bfloat16*>(qb + sw128_off(h, i_q + HALF, kNH)) =
              __float2bfloat16(x2 * qcs.x + x1 * qcs.y);
        }
        // R(delta) k for this thread's four rows, 8 pairs each: dims
        // 8ch..8ch+7 (first block) and their partners 64 + 8ch.. (second
        // block, same swizzled offset)
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
          const int rr = r0 + 32 * qq;
          const uint32_t off = rr * 128 + ((ch ^ (rr & 7)) << 4);
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

struct DTPlan {
  int n_whole, n_tail, n_ch;
  size_t cnt_bytes, po_bytes, ml_bytes, total;
};

// Items (batch element, KV head) are handed out whole for as many complete
// rounds of the grid as they fill (a chunk boundary costs the pipeline a few
// microseconds, so whole items are cheapest); the items of the last, partial
// round are cut into about grid / n_tail chunks each, so that every CTA
// takes a share of the tail.  At most one chunk per key tile of the longest
// item, and at most 64.
DTPlan dt_plan(int B, int Hq, int H, int T_loc, int m_cap) {
  DTPlan p{};
  const int64_t items = (int64_t)B * H;
  const int64_t tiles = ((int64_t)m_cap + kTK - 1) / kTK + (T_loc + kTK - 1) / kTK;
  const int64_t sms = std::max(1, num_sms());
  int64_t tail = items % sms;
  if (const char* e = std::getenv("MSA_DECODE_TAIL")) {  // tuning: cut items (-1 = all)
    const int v = std::atoi(e);
    if (v == -1) tail = items;
    else if (v >= 0 && v <= items) tail = v;
  }
  int64_t want = tail > 0 ? (sms + tail - 1) / tail : 1;
  if (const char* e = std::getenv("MSA_DECODE_CHUNKS")) {  // tuning: chunks per cut item
    const int v = std::atoi(e);
    if (v >= 1 && v <= 64) want = v;
  }
  p.n_ch = (int)std::max<int64_t>(1, std::min<int64_t>({want, tiles, 64}));
  if (p.n_ch == 1) tail = 0;  // nothing to cut
  p.n_tail = (int)tail;
  p.n_whole = (int)(items - tail);
  p.cnt_bytes = round_up((size_t)(1 + items) * sizeof(int), 256);
  const size_t rows = (size_t)tail * (Hq / H);
  p.po_bytes = tail ? round_up(rows * p.n_ch * kDim * sizeof(float), 256) : 0;
  p.ml_bytes = tail ? round_up(rows * p.n_ch * sizeof(float2), 256) : 0;
  p.total = p.cnt_bytes + p.po_bytes + p.ml_bytes;
  return p;
}

// (cos, sin) of p * w for an integer position p, the angle reduced modulo
// 2 pi in double on the host.
float2 host_cs(double p, double w) {
  const double two_pi = 6.283185307179586;
  const double th = p * w;
  const double r = th - std::nearbyint(th / two_pi) * two_pi;
  return make_float2((float)std::cos(r), (float)std::sin(r));
}

RopeTab rope_tab(float rope_base, int pos0, int T_loc) {
  RopeTab t;
  for (int i = 0; i < kDim / 2; ++i) {
    const double w = std::pow((double)rope_base, -2.0 * i / kDim);
    t.w[i] = (float)w;
    t.qpos[i] = host_cs((double)pos0 + T_loc - 1, w);
    t.qdelta[i] = host_cs((double)T_loc - 1, w);
    t.qstep[i] = host_cs((double)kTK, w);
  }
  return t;
}

template <int G>
int launch_dtc(int B, int T_loc, int Hq, int H, const void* q, const void* k_mem,
               const void* v_mem, const int32_t* mem_len, int m_cap, const void* k_loc,
               const void* v_loc, int pos0, float rope_base, float qscale, void* out, void* ws,
               cudaStream_t s, const FusedMemory* fm) {
  // fused: the memory is at most 8 * max_groups rows a query (for the plan)
  const int mem_rows_cap = fm ? 8 * fm->max_groups : m_cap;
  const DTPlan p = dt_plan(B, Hq, H, T_loc, mem_rows_cap);
  unsigned char* w = static_cast<unsigned char*>(ws);
  int* counters = reinterpret_cast<int*>(w);
  float* part_o = reinterpret_cast<float*>(w + p.cnt_bytes);
  float2* part_ml = reinterpret_cast<float2*>(w + p.cnt_bytes + p.po_bytes);
  CUtensorMap tkm, tvm, tkl, tvl;
  bool ok;
  if (fm) {  // the bank itself, 8-row boxes (one swizzle atom)
    ok = tma_map_sw128_bf16(&tkm, fm->k_bar, kDim, H, fm->n_chunks, 1, 8) &&
         tma_map_sw128_bf16(&tvm, fm->v_bar, kDim, H, fm->n_chunks, 1, 8);
  } else {
    const bool has_mem = m_cap > 0;
    const int64_t mem_rows = has_mem ? (int64_t)B * m_cap : (int64_t)B * T_loc;
    ok = tma_map_sw128_bf16(&tkm, has_mem ? k_mem : k_loc, kDim, H, mem_rows, 1, kTK) &&
         tma_map_sw128_bf16(&tvm, has_mem ? v_mem : v_loc, kDim, H, mem_rows, 1, kTK);
  }
  ok = ok && tma_map_sw128_bf16(&tkl, k_loc, kDim, H, (int64_t)B * T_loc, 1, kTK) &&
       tma_map_sw128_bf16(&tvl, v_loc, kDim, H, (int64_t)B * T_loc, 1, kTK);
  if (!ok) return note_cuda(cudaErrorInvalidValue);
  auto kern = fm ? attn_decode_tc_kernel<G, true> : attn_decode_tc_kernel<G, false>;
  int rc = ensure_smem_attr(reinterpret_cast<const void*>(kern), (int)DTS::ALLOC);
  if (rc) return rc;
  const int64_t n_chunks = (int64_t)p.n_whole + (int64_t)p.n_tail * p.n_ch;
  if (n_chunks > INT32_MAX) return MSA_ERR_UNSUPPORTED;
  // the chunk counter and the arrival counters start at zero on every call
  rc = note_cuda(cudaMemsetAsync(counters, 0, (size_t)(1 + p.n_tail) * sizeof(int), s));
  if (rc) return rc;
  const int grid = (int)std::min<int64_t>(n_chunks, num_sms());
  kern<<<grid, kTThreads, DTS::ALLOC, s>>>(
      tkm, tvm, tkl, tvl, T_loc, Hq, H, p.n_whole, p.n_tail, p.n_ch,
      static_cast<const __nv_bfloat16*>(q), fm ? fm->n_groups : mem_len, m_cap,
      fm ? fm->groups : nullptr, fm ? fm->max_groups : 0, rope_tab(rope_base, pos0, T_loc),
      qscale,
      counters, static_cast<__nv_bfloat16*>(out), part_o, part_ml, device_status_ptr());
  return check_launch();
}

int dispatch_dtc(int B, int T_loc, int Hq, int H, int D, const void* q, const void* k_mem,
                 const void* v_mem, const int32_t* mem_len, int m_cap, const void* k_loc,
                 const void* v_loc, int pos0, float rope_base, float qscale, void* out, void* ws,
                 cudaStream_t s, const FusedMemory* fm) {
  if (!aligned16(k_loc) || !aligned16(v_loc)) return MSA_ERR_INVALID_ARG;
  if (!fm && m_cap > 0 && (!aligned16(k_mem) || !aligned16(v_mem))) return MSA_ERR_INVALID_ARG;
  if (fm && (!aligned16(fm->k_bar) || !aligned16(fm->v_bar))) return MSA_ERR_INVALID_ARG;
  if ((int64_t)B * H > 65535 || (int64_t)B * std::max(m_cap, T_loc) > INT32_MAX)
    return MSA_ERR_UNSUPPORTED;
  const int G = Hq / H;
#define MSA_DTC_CASE(GG)                                                                    \
  if (D == kDim && G == GG)                                                                 \
    return launch_dtc<GG>(B, T_loc, Hq, H, q, k_mem, v_mem, mem_len, m_cap, k_loc, v_loc, \
                          pos0, rope_base, qscale, out, ws, s, fm);
  MSA_DTC_CASE(1) MSA_DTC_CASE(2) MSA_DTC_CASE(4) MSA_DTC_CASE(8) MSA_DTC_CASE(16)
#undef MSA_DTC_CASE
  return MSA_ERR_UNSUPPORTED;
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
  return dispatch_dtc(B, T_loc, Hq, H, D, q, k_mem, v_mem, mem_len, m_cap, k_loc, v_loc, pos0,
                      rope_base, qscale, out, ws, s, nullptr);
}

size_t attn_decode_tc_fused_workspace_size(int B, int T_loc, int Hq, int H, int max_groups) {
  return dt_plan(B, Hq, H, T_loc, 8 * max_groups).total;
}

int attn_decode_tc_launch_fused(int B, int T_loc, int Hq, int H, int D, const void* q,
                                const FusedMemory& fm, const void* k_loc, const void* v_loc,
                                int pos0, float rope_base, float qscale, void* out, void* ws,
                                cudaStream_t s) {
  return dispatch_dtc(B, T_loc, Hq, H, D, q, nullptr, nullptr, nullptr, 8 * fm.max_groups,
                      k_loc, v_loc, pos0, rope_base, qscale, out, ws, s, &fm);
}

}  // namespace msa
