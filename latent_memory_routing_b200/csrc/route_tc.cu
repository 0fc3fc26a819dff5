// bf16 routing scan on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Computes, for every chunk c of the pooled routing bank and every query b,
//   s[b,c] = max_t (1/H) sum_h cos(Q_r[b,t,h], K̄_r[c,h])
// and folds it into the document maximum -- "EverMind-AI/MSA: routing top-k
// compressed documents inside attention ..." (hysenlabs.com), §"Routing
// happens inside attention, not in a retrieval service in front of the model"
// (cosine similarity, mean over heads, token-wise maximum); the maximum over
// a document's chunks is this library's reading of the document score.
//
// Design.  The bank is streamed once per pass (<= 256 query columns):
//   * persistent CTAs, one per SM, each owning a contiguous range of
//     128-chunk tiles (so a tile's documents follow the previous tile's);
//   * warp 0 (one lane) TMA-loads the tile's K̄_r rows of one head (128 x 64
//     bf16 per K block, 128B-swizzled) and that head's normalised query
//     columns (N x 64) into a multi-stage shared-memory ring;
//   * raw bank: warps 2..5 (the transform, one thread per chunk row)
//     normalise each row in place -- |K̄_r[c,h]| from the row's 16-byte
//     pieces read in swizzled order (bank-conflict free), then
//     K̄_r / max(|K̄_r|, 1e-12) rounded to bf16 -- so a stage holds a whole
//     head.  Prepared bank (rows already unit-normalised by
//     msa_route_prepare_bank when the bank was built): no transform, and a
//     stage is one 64-wide K block, so twice as many stages fit;
//   * warp 1 (one lane) issues tcgen05.mma M=128 (chunks) x N (query
//     columns) x K=16 for every head and K block of the tile into ONE TMEM
//     accumulator: with unit rows on both sides (the query pre-normalised
//     with 1/H folded in) the sum over heads is the head-mean cosine; two
//     accumulators alternate between tiles so the next tile's MMAs overlap
//     this tile's epilogue;
//   * warps 6..9 (the epilogue, one thread per chunk row) find the row's
//     document from a window of chunk offsets prefetched during the previous
//     tile, read the 128 x N cosines from TMEM 32 columns at a time (the
//     next load in flight while one is reduced), take the maximum over each
//     query's tokens (a tree maximum when 32 columns belong to one query),
//     then over the rows of each document inside the warp (segmented
//     shuffle maximum), and issue one order-preserving atomicMax per
//     (query, document segment).  For queries of fewer than 32 tokens the
//     epilogue parks per-query maxima in shared memory and walks document
//     runs from a warp-uniform run mask instead (the column-owner epilogue);
//   * argmax mode (kArg, for the routing backward): the same scan keeps each
//     (query, document)'s first maximising (chunk, token) as a 64-bit key.
// Scores never round-trip through HBM.  No cluster multicast is used.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdlib>

#include "msa_common.cuh"
#include "route_tc.cuh"
#include "tc_ptx.cuh"

namespace msa {
namespace {

constexpr int kTile = 128;  // chunks per tile = MMA M = TMEM lanes
constexpr int kXWarps = 4;   // transform warps (raw bank)
constexpr int kEpiWarps = 4;
constexpr int kThreads = 64 + 32 * (kXWarps + kEpiWarps);
constexpr int kWindow = 256;  // documents cached per tile for chunk -> doc
constexpr int kEpiBar = 1;    // named barrier of the epilogue warps
constexpr int kMaxStages = 8;

// kPair: a CTA pair (cluster of 2, cta_group::2) shares each MMA -- M = 256
// chunks (128 per CTA), each CTA holding half of the N query columns -- so a
// CTA's stage carries half the query bytes (prepared bank, N = 256 only).
template <int N, int D, bool kPrep, bool kPair = false>
struct Cfg {
  static_assert(!kPair || (kPrep && N == 256), "pairs take the prepared bank, 256 columns");
  static constexpr int KB = D / 64;                   // 64-element K blocks per head
  static constexpr int SKB = kPrep ? 1 : KB;          // K blocks per stage
  static constexpr int SPH = KB / SKB;                // stages per head
  static constexpr int NB = kPair ? N / 2 : N;        // query columns in this CTA's stage
  static constexpr int A_BYTES = SKB * kTile * 128;
  static constexpr int B_BYTES = SKB * NB * 128;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int STAGES_FIT =
      (200 * 1024 - (N <= 128 ? kEpiWarps * (N * 33 + 32) * 4 : 0)) / STAGE;
  static constexpr int STAGES = STAGES_FIT > kMaxStages ? kMaxStages : STAGES_FIT;
  static constexpr int TMEM_COLS = 2 * N;
  static constexpr uint32_t IDESC = tc::idesc_bf16_f32(kPair ? 2 * kTile : kTile, N);
  // column-owner epilogue (queries of fewer than 32 tokens, N <= 128): per
  // epilogue warp, the warp's 32 rows x N per-query maxima, [slot][33]
  // (padded: row-wise writes and slot-wise reads both conflict-free), and
  // the 32 rows' document ids
  static constexpr int SCR_WORDS = N <= 128 ? N * 33 + 32 : 0;
  static constexpr size_t SCR = (size_t)kEpiWarps * SCR_WORDS * 4;
  static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE + SCR;
  static_assert(STAGES >= 2, "need a double-buffered ring");
  static_assert(N % 64 == 0 && N >= 64 && N <= 256, "N");
};

struct Aux {
  uint64_t full[kMaxStages], ready[kMaxStages], empty[kMaxStages], accf[2], acce[2];
  uint32_t tmem_base;
  int abort_flag;
  int d0;
  int64_t win[kWindow + 1];
};

__device__ __forceinline__ void epi_bar() {
  asm volatile("bar.sync %0, %1;" ::"n"(kEpiBar), "n"(32 * kEpiWarps) : "memory");
}

// x*x summed over the 8 bf16 of a 16-byte piece, in packed fp32 pairs.
__device__ __forceinline__ void sumsq8(const uint4& v, unsigned long long& acc) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const unsigned long long x =
        ((unsigned long long)(w[i] & 0xffff0000u) << 32) | (unsigned long long)(w[i] << 16);
    asm("fma.rn.f32x2 %0, %1, %1, %0;" : "+l"(acc) : "l"(x));
  }
}

__device__ __forceinline__ uint4 scale8(const uint4& v, unsigned long long k2) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const unsigned long long x =
        ((unsigned long long)(w[i] & 0xffff0000u) << 32) | (unsigned long long)(w[i] << 16);
    unsigned long long y;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(y) : "l"(x), "l"(k2));
    const float lo = __uint_as_float((uint32_t)y), hi = __uint_as_float((uint32_t)(y >> 32));
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    o[i] = *reinterpret_cast<uint32_t*>(&h);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// largest d in [0, n) with off[d] <= x, by bisection of a global array
__device__ __forceinline__ int bisect_global(const int64_t* off, int lo, int hi, int64_t x) {
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(off + mid) <= x) lo = mid; else hi = mid;
  }
  return lo;
}

// Per-row epilogue state shared by the reduction helpers.
struct Emit {
  const int64_t c;
  const int dd;
  const bool valid, head;
  const unsigned same;
  const int64_t C;
  const int n_docs;
  uint32_t* doc_u;
  uint32_t* chunk_u;
  __device__ __forceinline__ void operator()(float m, int b) const {
    const uint32_t o = valid ? f2o(m) : 0u;
    if (chunk_u && valid) atomicMax(chunk_u + (int64_t)b * C + c, o);
    uint32_t x = o;
#pragma unroll
    for (int k = 0; k < 5; ++k) {
      const uint32_t y = __shfl_down_sync(0xffffffffu, x, 1 << k);
      if (same & (1u << k)) x = max(x, y);
    }
    if (head) atomicMax(doc_u + (int64_t)b * n_docs + dd, x);
  }
};

// Folds 32 consecutive columns [cs, cs+32) of this row into the running
// token maximum m of query b (token t), emitting at each query's last
// column, at the last column of the pass (last_chunk) and at NT.
__device__ __forceinline__ void reduce32(const uint32_t (&r)[32], int cs, int NT, int T,
                                         bool last_chunk, float& m, int& b, int& t,
                                         const Emit& emit) {
  if (cs + 31 < NT && t + 32 <= T) {  // one query owns all 32 columns
    float v[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
      v[i] = fmaxf(__uint_as_float(r[i]), __uint_as_float(r[i + 16]));
#pragma unroll
    for (int w = 8; w; w >>= 1)
#pragma unroll
      for (int i = 0; i < w; ++i) v[i] = fmaxf(v[i], v[i + w]);
    m = fmaxf(m, v[0]);
    t += 32;
    if (t == T || last_chunk || cs + 32 >= NT) {
      emit(m, b);
      m = -INFINITY;
      if (t == T) { t = 0; ++b; }
    }
    return;
  }
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int col = cs + i;
    if (col >= NT) break;  // warp-uniform
    m = fmaxf(m, __uint_as_float(r[i]));
    if ((last_chunk && i == 31) || col + 1 >= NT || t + 1 == T) {
      emit(m, b);
      m = -INFINITY;
    }
    if (++t == T) { t = 0; ++b; }
  }
}

// kArg: instead of the document maximum, each (query, document) gets the
// 64-bit key of its first maximiser -- high word the order-preserving score,
// low word ~((chunk - document's first chunk) * T + token) -- so one
// atomicMax keeps the highest score, then the lowest chunk, then the lowest
// token (the host guarantees (chunks of a document) * T < 2^32).
template <int N, int D, bool kPrep, bool kPair, bool kArg>
__global__ void __launch_bounds__(kThreads, 1)
route_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
                int H, int NT, int T, int n_pass, int64_t C, int64_t n_tiles,
                const int64_t* __restrict__ coff, int n_docs, uint32_t* __restrict__ doc_u,
                uint32_t* __restrict__ chunk_u, unsigned long long* __restrict__ doc_key,
                int* __restrict__ status) {
  pdl_wait();  // launched as a programmatic dependent: nothing is touched before
  using K = Cfg<N, D, kPrep, kPair>;
  extern __shared__ __align__(1024) unsigned char smem_dyn[];
  __shared__ Aux aux;
  unsigned char* ring = tc::smem_align<1024>(smem_dyn);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // A unit is one 128-chunk tile, or for a CTA pair two adjacent tiles (the
  // even CTA takes the first); each CTA (pair) owns a contiguous unit range.
  const uint32_t crank = kPair ? tc::cluster_ctarank() : 0u;
  constexpr int kStep = kPair ? 2 : 1;  // tiles per unit
  const int64_t n_units = (n_tiles + kStep - 1) / kStep;
  const int64_t grp = blockIdx.x / kStep, n_grp = gridDim.x / kStep;
  const int64_t tb = grp * n_units / n_grp;
  const int64_t te = (grp + 1) * n_units / n_grp;
  auto unit_tile = [&](int64_t u) { return u * kStep + crank; };

  if (threadIdx.x == 0) {
    for (int i = 0; i < K::STAGES; ++i) {
      tc::mbar_init(&aux.full[i], 1);
      tc::mbar_init(&aux.ready[i], kXWarps);
      tc::mbar_init(&aux.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&aux.accf[i], 1);
      // a pair's leader waits for both CTAs' epilogue warps
      tc::mbar_init(&aux.acce[i], kEpiWarps * kStep);
    }
    aux.abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 1) {
    if constexpr (kPair) {
      tc::tmem_alloc_pair(&aux.tmem_base, K::TMEM_COLS);
      tc::tmem_relinquish_pair();
    } else {
      tc::tmem_alloc(&aux.tmem_base, K::TMEM_COLS);
      tc::tmem_relinquish();
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  // the peer's loads and arrivals target the leader's barriers: both CTAs'
  // barriers are initialised before either CTA goes on
  if constexpr (kPair) tc::cluster_sync();
  tc::tc_fence_after();
  const uint32_t tmem = aux.tmem_base;
  volatile int* abort_flag = &aux.abort_flag;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tc::tma_prefetch_desc(&tm_k);
      tc::tma_prefetch_desc(&tm_q);
      uint32_t u = 0;
      bool stop = false;
      for (int p = 0; p < n_pass && !stop; ++p)
        for (int64_t un = tb; un < te && !stop; ++un)
          for (int h = 0; h < H && !stop; ++h)
            for (int s = 0; s < K::SPH; ++s, ++u) {
              const int st = u % K::STAGES;
              const uint32_t ph = (u / K::STAGES) & 1u;
              if (*abort_flag || !tc::mbar_wait(&aux.empty[st], ph ^ 1u)) {
                record_error(status, MSA_ERR_TIMEOUT);
                *abort_flag = 1;
                stop = true;
                break;
              }
              const int64_t tile = unit_tile(un);
              unsigned char* a = ring + st * K::STAGE;
              unsigned char* b = a + K::A_BYTES;
              if constexpr (kPair) {
                // both CTAs' bytes count on the leader's barrier, which the
                // leader alone arms
                const uint32_t fb = tc::mapa_shared(&aux.full[st], 0);
                if (crank == 0) tc::mbar_arrive_expect_tx(&aux.full[st], 2 * K::STAGE);
                const int x = s * 64;
                tc::tma_load_3d_pair(a, &tm_k, fb, x, h, (int32_t)(tile * kTile));
                tc::tma_load_3d_pair(b, &tm_q, fb, x, p * N + (int)crank * K::NB, h);
              } else {
                tc::mbar_arrive_expect_tx(&aux.full[st], K::STAGE);
#pragma unroll
                for (int kb = 0; kb < K::SKB; ++kb) {
                  const int x = (s * K::SKB + kb) * 64;
                  tc::tma_load_3d(a + kb * kTile * 128, &tm_k, &aux.full[st], x, h,
                                  (int32_t)(tile * kTile));
                  tc::tma_load_3d(b + kb * N * 128, &tm_q, &aux.full[st], x, p * N, h);
                }
              }
            }
      // Drain: every load issued must have landed before the CTA exits (a
      // pair's loads, both CTAs', complete on the leader's barriers, and the
      // peer leaves only after the leader, at the closing cluster barrier).
      const uint32_t issued = u;
      if (crank == 0)
        for (uint32_t v = issued > (uint32_t)K::STAGES ? issued - K::STAGES : 0; v < issued; ++v)
          tc::mbar_wait(&aux.full[v % K::STAGES], (v / K::STAGES) & 1u);
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0 && crank == 0) {  // a pair's MMAs are issued by its leader
      uint32_t u = 0, it = 0;
      bool stop = false;
      // a pair's commits go to the barrier in each CTA
      const uint32_t peer_empty0 = kPair ? tc::mapa_shared(&aux.empty[0], 1) : 0u;
      const uint32_t peer_accf0 = kPair ? tc::mapa_shared(&aux.accf[0], 1) : 0u;
      for (int p = 0; p < n_pass && !stop; ++p)
        for (int64_t un = tb; un < te && !stop; ++un, ++it) {
          const int ab = it & 1;
          const uint32_t aph = (it >> 1) & 1u;
          const uint32_t d_tmem = tmem + ab * N;
          if (*abort_flag || !tc::mbar_wait(&aux.acce[ab], aph ^ 1u)) {
            record_error(status, MSA_ERR_TIMEOUT);
            *abort_flag = 1;
            break;
          }
          for (int h = 0; h < H && !stop; ++h)
            for (int s = 0; s < K::SPH; ++s, ++u) {
              const int st = u % K::STAGES;
              const uint32_t ph = (u / K::STAGES) & 1u;
              if (*abort_flag ||
                  !tc::mbar_wait(kPrep ? &aux.full[st] : &aux.ready[st], ph)) {
                record_error(status, MSA_ERR_TIMEOUT);
                *abort_flag = 1;
                stop = true;
                break;
              }
              tc::tc_fence_after();
              const uint64_t a_d = tc::sdesc_kmajor_sw128(tc::smem_u32(ring + st * K::STAGE));
              const uint64_t b_d = tc::desc_add(a_d, K::A_BYTES);
#pragma unroll
              for (int kk = 0; kk < K::SKB * 4; ++kk) {
                const uint32_t koff = (kk & 3) * 32;  // 16 bf16 = 32 B inside the swizzle atom
                const uint64_t ad = tc::desc_add(a_d, (kk >> 2) * (kTile * 128) + koff);
                const uint64_t bd = tc::desc_add(b_d, (kk >> 2) * (K::NB * 128) + koff);
                const uint32_t acc = (h > 0 || s > 0 || kk > 0) ? 1u : 0u;
                if constexpr (kPair) tc::mma_bf16_ss_pair(d_tmem, ad, bd, K::IDESC, acc);
                else tc::mma_bf16_ss(d_tmem, ad, bd, K::IDESC, acc);
              }
              if constexpr (kPair) {
                tc::mma_commit_pair(tc::smem_u32(&aux.empty[st]));
                tc::mma_commit_pair(peer_empty0 + st * (uint32_t)sizeof(uint64_t));
              } else {
                tc::mma_commit(&aux.empty[st]);
              }
            }
          if (!stop) {
            if constexpr (kPair) {
              tc::mma_commit_pair(tc::smem_u32(&aux.accf[ab]));
              tc::mma_commit_pair(peer_accf0 + ab * (uint32_t)sizeof(uint64_t));
            } else {
              tc::mma_commit(&aux.accf[ab]);
            }
          }
        }
    }
  } else if (warp < 2 + kXWarps) {
    // ------------------------------------------------ transform (raw bank)
    if (!kPrep) {
      const int row = (warp - 2) * 32 + lane;
      uint32_t u = 0;
      for (int p = 0; p < n_pass; ++p)
        for (int64_t tile = tb; tile < te; ++tile)
          for (int h = 0; h < H; ++h, ++u) {
            const int st = u % K::STAGES;
            const uint32_t ph = (u / K::STAGES) & 1u;
            // After a timeout every role keeps walking its loop without
            // waiting, so nobody blocks on a barrier that will not complete.
            if (!*abort_flag && !tc::mbar_wait(&aux.full[st], ph)) {
              record_error(status, MSA_ERR_TIMEOUT);
              *abort_flag = 1;
            }
            unsigned char* arow = ring + st * K::STAGE + row * 128;
            uint4 v[K::KB][8];
            unsigned long long ss2 = 0ull;
#pragma unroll
            for (int kb = 0; kb < K::KB; ++kb)
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                // piece j of the swizzled row sits at 16 * (j ^ row % 8); any
                // order serves a sum, and this one keeps the warp's 8-row
                // groups on distinct banks
                v[kb][j] = *reinterpret_cast<const uint4*>(arow + kb * (kTile * 128) +
                                                          ((j ^ (row & 7)) << 4));
                sumsq8(v[kb][j], ss2);
              }
            const float ss = __uint_as_float((uint32_t)ss2) + __uint_as_float((uint32_t)(ss2 >> 32));
            const float inv = 1.0f / fmaxf(sqrtf(ss), 1e-12f);
            const unsigned long long inv2 =
                ((unsigned long long)__float_as_uint(inv) << 32) | __float_as_uint(inv);
#pragma unroll
            for (int kb = 0; kb < K::KB; ++kb)
#pragma unroll
              for (int j = 0; j < 8; ++j)
                *reinterpret_cast<uint4*>(arow + kb * (kTile * 128) + ((j ^ (row & 7)) << 4)) =
                    scale8(v[kb][j], inv2);
            tc::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&aux.ready[st]);
          }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2 - kXWarps;
    const int quad = warp & 3;  // TMEM lane quarter this warp may access
    const int row = quad * 32 + lane;
    const int et = ew * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    uint32_t it = 0;
    for (int p = 0; p < n_pass; ++p) {
      const int col0 = p * N;
      // first tile of the pass: look its document window up synchronously
      if (tb < te) {
        if (ew == 0) {
          const int64_t d0 = warp_find_segment(coff, n_docs, unit_tile(tb) * kTile);
          if (lane == 0) aux.d0 = (int)d0;
        }
        epi_bar();
        const int d0 = aux.d0;
        for (int i = et; i <= kWindow; i += 32 * kEpiWarps) {
          const int64_t di = (int64_t)d0 + i;
          aux.win[i] = di <= n_docs ? __ldg(coff + di) : INT64_MAX;
        }
        epi_bar();
      }
      for (int64_t un = tb; un < te; ++un, ++it) {
        const int ab = it & 1;
        const uint32_t aph = (it >> 1) & 1u;
        const int64_t c0 = unit_tile(un) * kTile;
        const int64_t c = c0 + row;
        const int d0 = aux.d0;
        const int64_t wend = aux.win[kWindow];
        // this row's document (and, for kArg, the document's first chunk)
        int dd = -1;
        int64_t cdoc = 0;
        if (c < C) {
          if (c < wend) {
            int lo = 0, hi = kWindow;  // win[lo] <= c < win[hi]
            while (hi - lo > 1) {
              const int mid = (lo + hi) >> 1;
              if (aux.win[mid] <= c) lo = mid; else hi = mid;
            }
            dd = d0 + lo;
            if constexpr (kArg) cdoc = aux.win[lo];
          } else {  // more than kWindow documents in one tile (empty documents)
            dd = bisect_global(coff, d0, n_docs, c);
            if constexpr (kArg) cdoc = __ldg(coff + dd);
          }
        }
        // next tile's window: base document and prefetch into registers
        const bool has_next = un + 1 < te;
        int d0n = d0;
        int64_t w0 = INT64_MAX, w1 = INT64_MAX, w2 = INT64_MAX;
        if (has_next) {
          const int64_t cn = c0 + kStep * kTile;  // this CTA's next tile
          if (cn < wend) {
            int lo = 0, hi = kWindow;
            while (hi - lo > 1) {
              const int mid = (lo + hi) >> 1;
              if (aux.win[mid] <= cn) lo = mid; else hi = mid;
            }
            d0n = d0 + lo;
          } else {
            d0n = bisect_global(coff, d0, n_docs, cn);
          }
          if ((int64_t)d0n + et <= n_docs) w0 = __ldg(coff + d0n + et);
          if ((int64_t)d0n + et + 128 <= n_docs) w1 = __ldg(coff + d0n + et + 128);
          if (et == 0 && (int64_t)d0n + kWindow <= n_docs) w2 = __ldg(coff + d0n + kWindow);
        }
        const bool valid = dd >= 0;
        unsigned same = 0;  // segment structure of the warp's rows
#pragma unroll
        for (int k = 0; k < 5; ++k) {
          const int off = 1 << k;
          const int od = __shfl_down_sync(0xffffffffu, dd, off);
          if (lane + off < 32 && od == dd) same |= 1u << k;
        }
        const int up = __shfl_up_sync(0xffffffffu, dd, 1);
        const Emit emit{c, dd, valid, valid && (lane == 0 || up != dd), same, C, n_docs,
                        doc_u, chunk_u};

        if (!*abort_flag && !tc::mbar_wait(&aux.accf[ab], aph)) {
          record_error(status, MSA_ERR_TIMEOUT);
          *abort_flag = 1;
        }
        tc::tc_fence_after();
        const uint32_t tbase = tmem + lane_addr + ab * N;
        uint32_t r0[32], r1[32];
        if constexpr (kArg) {
          // First maximiser: per row and query, the best token (strictly
          // greater keeps the first); per document, the best row (the key
          // orders equal scores by chunk, then token).
          const uint32_t row_base = (uint32_t)((c - cdoc) * T);
          const bool head = emit.head;
          auto emit_arg = [&](float mm, int tt, int bb) {
            unsigned long long x =
                valid ? ((unsigned long long)f2o(mm) << 32) |
                            (unsigned long long)(0xffffffffu - (row_base + (uint32_t)tt))
                      : 0ull;
#pragma unroll
            for (int k = 0; k < 5; ++k) {
              const unsigned long long y = __shfl_down_sync(0xffffffffu, x, 1 << k);
              if (same & (1u << k)) x = x > y ? x : y;
            }
            if (head) atomicMax(doc_key + (int64_t)bb * n_docs + dd, x);
          };
          int b = col0 / T;
          int t = col0 - b * T;
          float m = -INFINITY;
          int mt = t;
          auto fold_arg = [&](const uint32_t (&r)[32], int cs, bool last_chunk) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int col = cs + i;
              if (col >= NT) break;  // warp-uniform
              const float v = __uint_as_float(r[i]);
              if (v > m) {
                m = v;
                mt = t;
              }
              if ((last_chunk && i == 31) || col + 1 >= NT || t + 1 == T) {
                emit_arg(m, mt, b);
                m = -INFINITY;
              }
              if (++t == T) {
                t = 0;
                ++b;
              }
            }
          };
          tc::tmem_ld32(tbase, r0);
          tc::tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < N / 32; j += 2) {
            if (j + 1 < N / 32) tc::tmem_ld32(tbase + (j + 1) * 32, r1);
            fold_arg(r0, col0 + j * 32, j + 1 == N / 32);
            tc::tmem_ld_wait();
            if (j + 1 < N / 32) {
              if (j + 2 < N / 32) tc::tmem_ld32(tbase + (j + 2) * 32, r0);
              fold_arg(r1, col0 + (j + 1) * 32, j + 2 == N / 32);
              tc::tmem_ld_wait();
            }
          }
          tc::tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if constexpr (kPair) tc::mbar_arrive_cluster(tc::mapa_shared(&aux.acce[ab], 0));
            else tc::mbar_arrive(&aux.acce[ab]);
          }
        } else if (K::SCR_WORDS > 0 && T < 32) {
          // Column-owner epilogue.  (1) each row folds its columns into one
          // maximum per query (slot) and parks it in shared memory, which
          // frees the accumulator at once; (2) lane s owns slot s (s + 32,
          // ...) and walks the warp's 32 rows in chunk order -- a
          // document's rows are one run -- with one atomicMax per run.
          uint32_t* scr = reinterpret_cast<uint32_t*>(ring + K::STAGES * K::STAGE) +
                          ew * K::SCR_WORDS;
          int* dw = reinterpret_cast<int*>(scr + N * 33);
          dw[lane] = dd;
          const int col_end = min(col0 + N, NT);
          const int b_first = col0 / T;
          int tq = col0 - b_first * T;  // token of the current query
          int slot = 0;
          float m = -INFINITY;
          auto fold32 = [&](const uint32_t (&r)[32], int cs) {
            if (T == 1) {
              // one query per column: every column is parked as it is, with
              // no loop-carried state (independent stores)
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const int col = cs + i;
                if (col < col_end) {  // warp-uniform
                  const uint32_t o = valid ? f2o(__uint_as_float(r[i])) : 0u;
                  scr[(col - col0) * 33 + lane] = o;
                  if (chunk_u && valid) atomicMax(chunk_u + (int64_t)col * C + c, o);
                }
              }
              return;
            }
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int col = cs + i;
              if (col >= col_end) break;  // warp-uniform
              m = fmaxf(m, __uint_as_float(r[i]));
              if (++tq == T || col + 1 == col_end) {
                const uint32_t o = valid ? f2o(m) : 0u;
                scr[slot * 33 + lane] = o;
                if (chunk_u && valid) atomicMax(chunk_u + (int64_t)(b_first + slot) * C + c, o);
                m = -INFINITY;
                if (tq == T) {
                  tq = 0;
                  ++slot;
                }
              }
            }
          };
          tc::tmem_ld32(tbase, r0);
          tc::tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < N / 32; j += 2) {
            if (j + 1 < N / 32) tc::tmem_ld32(tbase + (j + 1) * 32, r1);
            fold32(r0, col0 + j * 32);
            tc::tmem_ld_wait();
            if (j + 1 < N / 32) {
              if (j + 2 < N / 32) tc::tmem_ld32(tbase + (j + 2) * 32, r0);
              fold32(r1, col0 + (j + 1) * 32);
              tc::tmem_ld_wait();
            }
          }
          tc::tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if constexpr (kPair) tc::mbar_arrive_cluster(tc::mapa_shared(&aux.acce[ab], 0));
            else tc::mbar_arrive(&aux.acce[ab]);
          }
          const int n_slots = (col_end - 1) / T - b_first + 1;
          // the warp's document runs are the same for every slot: bit rr of
          // `heads` marks a row that starts one (warp-uniform branches below)
          const unsigned heads = __ballot_sync(0xffffffffu, lane == 0 || up != dd);
          for (int sl = lane; sl < n_slots; sl += 32) {
            uint32_t* doc_row = doc_u + (int64_t)(b_first + sl) * n_docs;
            const uint32_t* v = scr + sl * 33;
            uint32_t vals[32];
#pragma unroll
            for (int rr = 0; rr < 32; ++rr) vals[rr] = v[rr];  // all loads first
            int cd = dw[0];
            uint32_t cur = vals[0];
#pragma unroll
            for (int rr = 1; rr < 32; ++rr) {
              if ((heads >> rr) & 1u) {
                if (cd >= 0) atomicMax(doc_row + cd, cur);
                cd = dw[rr];
                cur = vals[rr];
              } else {
                cur = max(cur, vals[rr]);
              }
            }
            if (cd >= 0) atomicMax(doc_row + cd, cur);
          }
          __syncwarp();  // the next tile rewrites scr and dw
        } else {
          int b = col0 / T;
          int t = col0 - b * T;
          float m = -INFINITY;
          tc::tmem_ld32(tbase, r0);
          tc::tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < N / 32; j += 2) {
            if (j + 1 < N / 32) tc::tmem_ld32(tbase + (j + 1) * 32, r1);
            reduce32(r0, col0 + j * 32, NT, T, j + 1 == N / 32, m, b, t, emit);
            tc::tmem_ld_wait();
            if (j + 1 < N / 32) {
              if (j + 2 < N / 32) tc::tmem_ld32(tbase + (j + 2) * 32, r0);
              reduce32(r1, col0 + (j + 1) * 32, NT, T, j + 2 == N / 32, m, b, t, emit);
              tc::tmem_ld_wait();
            }
          }
          tc::tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if constexpr (kPair) tc::mbar_arrive_cluster(tc::mapa_shared(&aux.acce[ab], 0));
            else tc::mbar_arrive(&aux.acce[ab]);
          }
        }
        epi_bar();  // everyone is done with this tile's window
        if (has_next) {
          aux.win[et] = w0;
          aux.win[et + 128] = w1;
          if (et == 0) {
            aux.win[kWindow] = w2;
            aux.d0 = d0n;
          }
        }
        epi_bar();
      }
    }
  }

  pdl_trigger();  // the scan's work is issued: the next kernel may be scheduled
  tc::tc_fence_before();
  __syncthreads();
  // neither CTA of a pair frees TMEM or leaves while the other may still
  // signal its barriers
  if constexpr (kPair) tc::cluster_sync();
  if (warp == 1) {
    tc::tc_fence_after();
    if constexpr (kPair) tc::tmem_dealloc_pair(tmem, K::TMEM_COLS);
    else tc::tmem_dealloc(tmem, K::TMEM_COLS);
  }
}

// Prepared routing bank: each (chunk, head) row divided by max(|row|, 1e-12)
// and rounded to bf16.  Two rows per warp, 16 lanes x 16 bytes per row.
template <int D>
__global__ void __launch_bounds__(256)
prepare_bank_kernel(int64_t n_rows, const __nv_bfloat16* __restrict__ src,
                    __nv_bfloat16* __restrict__ dst) {
  constexpr int LPR = D / 8;  // lanes per row
  const int64_t gt = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t row = gt / LPR;
  const int sub = (int)(gt % LPR);
  const bool live = row < n_rows;
  uint4 v = make_uint4(0, 0, 0, 0);
  if (live) v = ld_stream16(src + row * D + sub * 8);
  float f[8];
  Vec16<__nv_bfloat16>::unpack(v, f);
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) ss = fmaf(f[i], f[i], ss);
#pragma unroll
  for (int o = LPR / 2; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float inv = 1.0f / fmaxf(sqrtf(ss), 1e-12f);
#pragma unroll
  for (int i = 0; i < 8; ++i) f[i] *= inv;
  if (live) st16(dst + row * D + sub * 8, Vec16<__nv_bfloat16>::pack(f));
}

// ----------------------------------------------------------------- host

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
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

// 3-D bf16 tensor map, dims (inner first) {d0, d1, d2}, box {64, b1, b2},
// 128-byte swizzle, zero fill out of bounds.
bool make_map(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
              uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t b1, uint32_t b2) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
  const cuuint32_t box[3] = {64, b1, b2};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int N, int D, bool kPrep, bool kPair = false, bool kArg = false>
int launch(int B, int T, int H, const __nv_bfloat16* qhat, int n_pad, const __nv_bfloat16* kr,
           int64_t C, const int64_t* coff, int n_docs, uint32_t* doc_u, uint32_t* chunk_u,
           unsigned long long* doc_key, int* status, cudaStream_t s) {
  using K = Cfg<N, D, kPrep, kPair>;
  CUtensorMap tm_k, tm_q;
  if (!make_map(&tm_k, kr, D, H, C, (uint64_t)D * 2, (uint64_t)H * D * 2, 1, kTile))
    return note_cuda(cudaErrorInvalidValue);
  if (!make_map(&tm_q, qhat, D, n_pad, H, (uint64_t)D * 2, (uint64_t)n_pad * D * 2, K::NB, 1))
    return note_cuda(cudaErrorInvalidValue);
  auto kern = route_tc_kernel<N, D, kPrep, kPair, kArg>;
  int rc = ensure_smem_attr(reinterpret_cast<const void*>(kern), (int)K::SMEM);
  if (rc) return rc;
  const int64_t n_tiles = (C + kTile - 1) / kTile;
  const int NT = B * T;
  const int n_pass = n_pad / N;
  if constexpr (kPair) {
    // one CTA pair per TPC (two SMs), each pair a contiguous range of
    // 256-chunk units
    const int64_t n_units = (n_tiles + 1) / 2;
    const int pairs = (int)std::min<int64_t>(n_units, std::max(1, num_sms() / 2));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * pairs));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = K::SMEM;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // see pdl_wait
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return note_cuda(cudaLaunchKernelEx(&cfg, kern, tm_k, tm_q, H, NT, T, n_pass, C, n_tiles,
                                        coff, n_docs, doc_u, chunk_u, doc_key, status));
  } else {
    const int grid = (int)std::min<int64_t>(n_tiles, num_sms());
    return launch_pdl(kern, dim3(grid), dim3(kThreads), K::SMEM, s, tm_k, tm_q, H, NT, T, n_pass,
                      C, n_tiles, coff, n_docs, doc_u, chunk_u, doc_key, status);
  }
}

}  // namespace

int64_t route_tc_columns(int64_t nt) {
  if (nt <= 64) return 64;
  if (nt <= 128) return 128;
  return (nt + 255) / 256 * 256;
}

int route_tc_launch(int B, int T, int H, int D, const __nv_bfloat16* qhat, int n_pad,
                    const __nv_bfloat16* kr, int64_t C, const int64_t* coff, int n_docs,
                    uint32_t* doc_u, uint32_t* chunk_u, int* status, bool prepared,
                    cudaStream_t s) {
  const int N = n_pad <= 128 ? n_pad : 256;
  if (!aligned16(qhat) || !aligned16(kr)) return MSA_ERR_INVALID_ARG;
  // a prepared bank at 256 columns runs on CTA pairs unless MSA_ROUTE_PAIRS=0
  // asks for the single-CTA kernel (both compute the same scores)
  static const bool pairs = [] {
    const char* e = getenv("MSA_ROUTE_PAIRS");
    return !(e && e[0] == '0');
  }();
  if (prepared && N == 256 && pairs) {
    if (D == 128)
      return launch<256, 128, true, true>(B, T, H, qhat, n_pad, kr, C, coff, n_docs, doc_u,
                                          chunk_u, nullptr, status, s);
    if (D == 64)
      return launch<256, 64, true, true>(B, T, H, qhat, n_pad, kr, C, coff, n_docs, doc_u,
                                         chunk_u, nullptr, status, s);
  }
#define MSA_ROUTE_CASE(NN, DD, PP)                                                        \
  if (N == NN && D == DD && prepared == PP)                                                \
    return launch<NN, DD, PP>(B, T, H, qhat, n_pad, kr, C, coff, n_docs, doc_u, chunk_u, \
                              nullptr, status, s);
  MSA_ROUTE_CASE(64, 64, false)
  MSA_ROUTE_CASE(64, 128, false)
  MSA_ROUTE_CASE(128, 64, false)
  MSA_ROUTE_CASE(128, 128, false)
  MSA_ROUTE_CASE(256, 64, false)
  MSA_ROUTE_CASE(256, 128, false)
  MSA_ROUTE_CASE(64, 64, true)
  MSA_ROUTE_CASE(64, 128, true)
  MSA_ROUTE_CASE(128, 64, true)
  MSA_ROUTE_CASE(128, 128, true)
  MSA_ROUTE_CASE(256, 64, true)
  MSA_ROUTE_CASE(256, 128, true)
#undef MSA_ROUTE_CASE
  return MSA_ERR_UNSUPPORTED;
}

int route_tc_argmax_launch(int B, int T, int H, int D, const __nv_bfloat16* qhat, int n_pad,
                           const __nv_bfloat16* kr, int64_t C, const int64_t* coff, int n_docs,
                           unsigned long long* doc_key, int* status, cudaStream_t s) {
  const int N = n_pad <= 128 ? n_pad : 256;
  if (!aligned16(qhat) || !aligned16(kr)) return MSA_ERR_INVALID_ARG;
#define MSA_ARG_CASE(NN, DD)                                                             \
  if (N == NN && D == DD)                                                                 \
    return launch<NN, DD, false, false, true>(B, T, H, qhat, n_pad, kr, C, coff, n_docs, \
                                              nullptr, nullptr, doc_key, status, s);
  MSA_ARG_CASE(64, 64)
  MSA_ARG_CASE(64, 128)
  MSA_ARG_CASE(128, 64)
  MSA_ARG_CASE(128, 128)
  MSA_ARG_CASE(256, 64)
  MSA_ARG_CASE(256, 128)
#undef MSA_ARG_CASE
  return MSA_ERR_UNSUPPORTED;
}

int route_prepare_bank_launch(int64_t n_rows, int D, const __nv_bfloat16* src,
                              __nv_bfloat16* dst, cudaStream_t s) {
  const int64_t threads = n_rows * (D / 8);
  const int64_t blocks = (threads + 255) / 256;
  if (blocks > 0x7fffffffLL) return MSA_ERR_UNSUPPORTED;
  if (D == 64)
    prepare_bank_kernel<64><<<(unsigned)blocks, 256, 0, s>>>(n_rows, src, dst);
  else
    prepare_bank_kernel<128><<<(unsigned)blocks, 256, 0, s>>>(n_rows, src, dst);
  return check_launch();
}

}  // namespace msa
