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
// Design (HBM-bound: every K/V byte is read once, so the kernel is built to
// keep loads in flight and spend few instructions per key).  One CTA of 256
// threads per (key split, batch element, KV head) serves the G query heads
// that share the KV head.  The CTA walks its share of the key tiles -- the
// memory rows [0, M) in 64-row tiles, then the local rows [0, T_loc) in
// 64-row tiles, so no tile mixes the two:
//   * one thread issues one TMA load per tile for K and one for V (64 rows of
//     this head, 256 bytes each, stored densely) into a 3-stage ring with an
//     mbarrier per stage; the stage freed by the previous tile is refilled
//     right after the first block barrier of the next;
//   * RoPE, relative form: a local key at tile offset delta (0..63) of the
//     tile whose first key sits Delta positions before the query satisfies
//     <R(p_q) q, R(p_k) k> = <R(Delta) q, R(delta) k>.  Each thread keeps the
//     (cos, sin) of its two fixed row offsets delta in registers and rotates
//     the K row it reads; the query is rotated once per tile by Delta (its
//     (cos, sin) advance by one complex step of -64 positions per tile from
//     an exact anchor).  Memory keys are not rotated and meet R(p_q) q;
//   * Q K: eight threads per key row, eight rotate-half pairs each, packed
//     fp32 FMAs against the rotated, scaled queries in shared memory, then a
//     three-step shuffle sum;
//   * softmax: one warp per query head over the tile's 64 scores (base-2
//     exponent domain), writing p twice, as a packed pair, for P V;
//   * P V: warp w takes keys w, w+8, ...; lane l owns dims 4l..4l+3 of every
//     head, so one V load feeds all G heads and no shuffles are needed; the
//     eight warps' partial O are summed once, at the end, in shared memory;
//   * splits write (max, sum, O) partials that the split-KV combine kernel
//     merges; a single split writes the normalised output directly.
#include <cudaTypedefs.h>

#include <algorithm>

#include "attn_tc.cuh"
#include "msa_common.cuh"
#include "tc_ptx.cuh"

namespace msa {
namespace {

constexpr int kDThreads = 256;
constexpr int kDWarps = kDThreads / 32;
constexpr int kDKeys = 64;                   // keys per tile
constexpr int kDStages = 3;
constexpr int kDParts = 8;                   // threads per key row in Q K
constexpr int kDRows = kDThreads / kDParts;  // rows per Q K pass
constexpr int kDD = 128;                     // head dim
constexpr int kDRowB = kDD * 2;
constexpr int kDTileB = kDKeys * kDRowB;     // one K or V tile
constexpr int kDStageB = 2 * kDTileB;
constexpr int kScStride = kDKeys + 4;        // score rows padded against bank conflicts

template <int G>
struct DSmem {
  // dynamic shared memory, offsets from a 128-byte aligned base
  static constexpr size_t RING = 0;                                  // [stage][K|V][64][128] bf16
  static constexpr size_t QRAW = RING + (size_t)kDStages * kDStageB;  // [G][D] f32, scaled
  static constexpr size_t QMEM = QRAW + (size_t)G * kDD * 4;          // [G][qperm(D)] R(p_q) q
  static constexpr size_t QT = QMEM + (size_t)G * kDD * 4;            // [2][G][qperm(D)] R(Delta) q
  static constexpr size_t SC = QT + 2 * (size_t)G * kDD * 4;          // [2][G][kScStride] scores
  static constexpr size_t PP = SC + 2 * (size_t)G * kScStride * 4;    // [2][64][G] (p, p)
  static constexpr size_t AL = PP + 2 * (size_t)kDKeys * G * 8;       // [2][G] alpha
  static constexpr size_t ML = AL + 2 * (size_t)G * 4;                // [G] (m, l)
  static constexpr size_t BAR = (ML + (size_t)G * 8 + 7) & ~size_t(7);  // [stages] mbarriers
  static constexpr size_t WF = BAR + kDStages * 8;                    // [64] inverse freqs (f64)
  static constexpr size_t CS = WF + (size_t)(kDD / 2) * 8;            // [2][64] e^{i 32 w}, e^{i 64 w}
  static constexpr size_t FLAG = CS + 2 * (size_t)(kDD / 2) * 8;      // abort flag
  static constexpr size_t ALLOC = FLAG + 16 + 128;  // + alignment slack
  // the cross-warp O reduction reuses the ring: [warp][G][D] f32
  static_assert((size_t)kDWarps * G * kDD * 4 <= (size_t)kDStages * kDStageB, "reduction fits");
};

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ unsigned long long pk2(float lo, float hi) {
  return (unsigned long long)__float_as_uint(lo) | ((unsigned long long)__float_as_uint(hi) << 32);
}
__device__ __forceinline__ float lo2(unsigned long long v) { return __uint_as_float((uint32_t)v); }
__device__ __forceinline__ float hi2(unsigned long long v) {
  return __uint_as_float((uint32_t)(v >> 32));
}
// o += a * b on packed fp32 pairs
__device__ __forceinline__ void fma2(unsigned long long& o, unsigned long long a,
                                     unsigned long long b) {
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(o) : "l"(a), "l"(b));
}
__device__ __forceinline__ unsigned long long mul2(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ unsigned long long add2(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// Shared-memory position of dim d in a stored query row: [chunk][part][4]
// with part = (d mod 64) / 8 and chunk = 2 (d >= 64) + (d mod 8) / 4, so the
// eight Q K parts of a row read one contiguous 128-byte line per chunk.
__device__ __forceinline__ int qperm(int d) {
  const int dd = d & 63;
  return ((d >> 6) * 2 + ((dd & 7) >> 2)) * 32 + (dd >> 3) * 4 + (dd & 3);
}
// One halving step of a reduce-scatter over the lanes that differ in bit
// `mask` of their part index: of N values, the lane with the bit clear keeps
// the lower half and sends the upper half, its partner the reverse; each
// keeps the sum of its half.  Returns the offset of the kept half.
template <int N>
__device__ __forceinline__ int rs_halve(float (&v)[N], int mask, bool up) {
#pragma unroll
  for (int i = 0; i < N / 2; ++i) {
    const float send = up ? v[i] : v[i + N / 2];
    const float keep = up ? v[i + N / 2] : v[i];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, mask);
  }
  return up ? N / 2 : 0;
}
// Sums G per-lane values over the 8 lanes of a Q K row group.  On return the
// lane holds the complete sums of heads base .. base + max(G/8, 1) - 1 in
// v[0 ..], base returned; for G < 8 neighbouring lanes hold duplicates.
template <int G>
__device__ __forceinline__ int reduce_scatter8(float (&v)[G], int part) {
  int base = 0;
  constexpr int N1 = G >= 2 ? G / 2 : 1, N2 = N1 >= 2 ? N1 / 2 : 1;
  if constexpr (G >= 2) base += rs_halve<G>(v, 4, part & 4);
  else v[0] += __shfl_xor_sync(0xffffffffu, v[0], 4);
  if constexpr (N1 >= 2) base += rs_halve<N1>(*reinterpret_cast<float(*)[N1]>(v), 2, part & 2);
  else v[0] += __shfl_xor_sync(0xffffffffu, v[0], 2);
  if constexpr (N2 >= 2) base += rs_halve<N2>(*reinterpret_cast<float(*)[N2]>(v), 1, part & 1);
  else v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1);
  return base;
}

// two bf16 (lo, hi halves of w) -> packed fp32 pair
__device__ __forceinline__ unsigned long long bf2_to_f2(uint32_t w) {
  return ((unsigned long long)(w & 0xffff0000u) << 32) | (unsigned long long)(w << 16);
}

template <int G>
__global__ void __launch_bounds__(kDThreads, G <= 4 ? 2 : 1)
attn_decode_kernel(const __grid_constant__ CUtensorMap tm_km,
                   const __grid_constant__ CUtensorMap tm_vm,
                   const __grid_constant__ CUtensorMap tm_kl,
                   const __grid_constant__ CUtensorMap tm_vl, int T_loc, int Hq, int H,
                   const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ mem_len,
                   int m_cap, int64_t pos0, double base, float qscale, int n_split,
                   __nv_bfloat16* __restrict__ out, float* __restrict__ part_o,
                   float2* __restrict__ part_ml, int* __restrict__ status) {
  using S = DSmem<G>;
  constexpr int HALF = kDD / 2;
  constexpr int NH = G < kDWarps ? G : kDWarps;  // softmax warps
  constexpr int HPW = G / NH;                    // heads per softmax warp
  extern __shared__ __align__(128) unsigned char dsm_raw[];
  unsigned char* sm = tc::smem_align<128>(dsm_raw);
  unsigned char* ring = sm + S::RING;
  float* qraw = reinterpret_cast<float*>(sm + S::QRAW);
  float* qmem = reinterpret_cast<float*>(sm + S::QMEM);
  float* qt = reinterpret_cast<float*>(sm + S::QT);
  float* sc = reinterpret_cast<float*>(sm + S::SC);
  unsigned long long* pp = reinterpret_cast<unsigned long long*>(sm + S::PP);
  float* al = reinterpret_cast<float*>(sm + S::AL);
  float2* mlw = reinterpret_cast<float2*>(sm + S::ML);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + S::BAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + S::FLAG);

  const int split = blockIdx.x;
  const int b = blockIdx.y / H, g = blockIdx.y % H;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int M = min(max(mem_len[b], 0), m_cap);
  const int n_mt = (M + kDKeys - 1) / kDKeys;
  const int n_all = n_mt + (T_loc + kDKeys - 1) / kDKeys;
  const int j_lo = (int)((int64_t)split * n_all / n_split);
  const int j_hi = (int)((int64_t)(split + 1) * n_all / n_split);
  const int nt = j_hi - j_lo;
  if (nt <= 0) {  // an empty split (more splits than tiles): neutral partial
    for (int e = tid; e < G * kDD; e += kDThreads) {
      const int64_t row_id = (int64_t)b * Hq + g * G + e / kDD;
      part_o[(row_id * n_split + split) * kDD + e % kDD] = 0.f;
      if (e % kDD == 0) part_ml[row_id * n_split + split] = make_float2(-INFINITY, 0.f);
    }
    return;
  }

  // tile jj of the (b, g) key list: memory tiles first, then local tiles
  auto tile_mem = [&](int jj) { return jj < n_mt; };
  auto tile_key0 = [&](int jj) { return jj < n_mt ? jj * kDKeys : (jj - n_mt) * kDKeys; };
  auto tile_valid = [&](int jj) {
    return jj < n_mt ? min(kDKeys, M - jj * kDKeys) : min(kDKeys, T_loc - (jj - n_mt) * kDKeys);
  };
  auto issue = [&](int j) {  // thread 0: TMA loads of relative tile j
    const int st = j % kDStages, jj = j_lo + j;
    unsigned char* kd = ring + (size_t)st * kDStageB;
    tc::mbar_arrive_expect_tx(&full[st], kDStageB);
    if (tile_mem(jj)) {
      const int row = b * m_cap + tile_key0(jj);
      tc::tma_load_3d(kd, &tm_km, &full[st], 0, g, row);
      tc::tma_load_3d(kd + kDTileB, &tm_vm, &full[st], 0, g, row);
    } else {
      const int row = b * T_loc + tile_key0(jj);
      tc::tma_load_3d(kd, &tm_kl, &full[st], 0, g, row);
      tc::tma_load_3d(kd + kDTileB, &tm_vl, &full[st], 0, g, row);
    }
  };

  if (tid == 0) {
    for (int i = 0; i < kDStages; ++i) tc::mbar_init(&full[i], 1);
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  __syncthreads();
  int issued = 0;
  if (tid == 0)
    for (; issued < kDStages - 1 && issued < nt; ++issued) issue(issued);

  // raw query of the group, scaled (qscale folds 1/sqrt(D) and log2 e)
  for (int e = tid; e < G * kDD; e += kDThreads)
    qraw[e] = __bfloat162float(q[((int64_t)b * Hq + g * G) * kDD + e]) * qscale;

  // per-pair tables, once per CTA: inverse frequency w_i, e^{i 32 w_i} and
  // e^{i 64 w_i}
  double* wf = reinterpret_cast<double*>(sm + S::WF);
  float2* cs32 = reinterpret_cast<float2*>(sm + S::CS);
  float2* cs64 = cs32 + HALF;
  if (tid < HALF) {
    const double w = rope_inv_freq(base, tid, kDD);
    wf[tid] = w;
    cs32[tid] = rope_cs(kDRows, w);
    cs64[tid] = rope_cs(kDKeys, w);
  }
  __syncthreads();  // qraw and the tables ready

  // per-thread RoPE state
  const int i_q = tid % HALF;  // pair index this thread rotates the query on
  const double wq = wf[i_q];
  const int row = tid / kDParts, part = tid % kDParts;  // Q K: row, 8-pair part
  float kc[2][8], ks[2][8];  // (cos, sin) of delta = row, row + 32
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float2 c0 = rope_cs(row, wf[part * 8 + e]), st = cs32[part * 8 + e];
    kc[0][e] = c0.x;
    ks[0][e] = c0.y;
    kc[1][e] = c0.x * st.x - c0.y * st.y;  // delta + 32: one complex product
    ks[1][e] = c0.y * st.x + c0.x * st.y;
  }
  if (n_mt > j_lo) {  // R(p_q) q for the memory tiles
    const float2 c = rope_cs(pos0 + T_loc - 1, wq);
    for (int e = tid; e < G * HALF; e += kDThreads) {
      const int h = e / HALF;
      const float x1 = qraw[h * kDD + i_q], x2 = qraw[h * kDD + i_q + HALF];
      qmem[h * kDD + qperm(i_q)] = x1 * c.x - x2 * c.y;
      qmem[h * kDD + qperm(i_q + HALF)] = x2 * c.x + x1 * c.y;
    }
  }
  // R(Delta) q for local tiles: exact anchor at the first local tile, then
  // one step of -64 positions per tile
  float2 qcs = make_float2(1.f, 0.f);
  const float2 qstep = cs64[i_q];
  bool anchored = false;
  auto make_qt = [&](int j) {
    const int jj = j_lo + j;
    if (tile_mem(jj)) return;
    const int Delta = T_loc - 1 - tile_key0(jj);
    if (!anchored) {
      qcs = rope_cs(Delta, wq);
      anchored = true;
    } else {  // multiply by e^{-i 64 w}
      const float c = qcs.x * qstep.x + qcs.y * qstep.y;
      qcs.y = qcs.y * qstep.x - qcs.x * qstep.y;
      qcs.x = c;
    }
    float* dst = qt + (j & 1) * G * kDD;
    for (int e = tid; e < G * HALF; e += kDThreads) {
      const int h = e / HALF;
      const float x1 = qraw[h * kDD + i_q], x2 = qraw[h * kDD + i_q + HALF];
      dst[h * kDD + qperm(i_q)] = x1 * qcs.x - x2 * qcs.y;
      dst[h * kDD + qperm(i_q + HALF)] = x2 * qcs.x + x1 * qcs.y;
    }
  };
  make_qt(0);
  __syncthreads();  // qmem and the first qt ready

  float m_run[HPW], l_run[HPW];  // softmax warps: per head
#pragma unroll
  for (int a = 0; a < HPW; ++a) {
    m_run[a] = -INFINITY;
    l_run[a] = 0.f;
  }
  unsigned long long acc[G][2];  // P V: dims 4 lane .. +3 of each head
#pragma unroll
  for (int h = 0; h < G; ++h) acc[h][0] = acc[h][1] = 0ull;

  for (int j = 0; j < nt; ++j) {
    const int st = j % kDStages, jj = j_lo + j;
    const bool mem = tile_mem(jj);
    const int n_valid = tile_valid(jj);
    if (!tc::mbar_wait(&full[st], (j / kDStages) & 1)) {
      record_error(status, MSA_ERR_TIMEOUT);
      *abort_flag = 1;
    }
    const unsigned char* kt = ring + (size_t)st * kDStageB;
    const unsigned char* vt = kt + kDTileB;
    const float* qb = mem ? qmem : qt + (j & 1) * G * kDD;
    float* scb = sc + (j & 1) * G * kScStride;

    // ---- Q K
#pragma unroll
    for (int pass = 0; pass < kDKeys / kDRows; ++pass) {
      const int r = row + pass * kDRows;
      unsigned long long sacc[G];
#pragma unroll
      for (int h = 0; h < G; ++h) sacc[h] = 0ull;
      if (r < n_valid) {
        const uint4 w1 = *reinterpret_cast<const uint4*>(kt + r * kDRowB + part * 16);
        const uint4 w2 = *reinterpret_cast<const uint4*>(kt + r * kDRowB + HALF * 2 + part * 16);
        const uint32_t a1[4] = {w1.x, w1.y, w1.z, w1.w}, a2[4] = {w2.x, w2.y, w2.z, w2.w};
        unsigned long long y1[4], y2[4];  // pairs (2u, 2u+1) of each half
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          y1[u] = bf2_to_f2(a1[u]);
          y2[u] = bf2_to_f2(a2[u]);
        }
        if (!mem) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const unsigned long long c2 = pk2(kc[pass][2 * u], kc[pass][2 * u + 1]);
            const unsigned long long s2 = pk2(ks[pass][2 * u], ks[pass][2 * u + 1]);
            const unsigned long long ns2 = pk2(-ks[pass][2 * u], -ks[pass][2 * u + 1]);
            unsigned long long n1 = mul2(y1[u], c2), n2 = mul2(y2[u], c2);
            fma2(n1, y2[u], ns2);  // x1 c - x2 s
            fma2(n2, y1[u], s2);   // x2 c + x1 s
            y1[u] = n1;
            y2[u] = n2;
          }
        }
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float* qh = qb + h * kDD + part * 4;  // chunks at +0, 32, 64, 96
          const ulonglong2 qa = *reinterpret_cast<const ulonglong2*>(qh);
          const ulonglong2 qe = *reinterpret_cast<const ulonglong2*>(qh + 32);
          const ulonglong2 qc = *reinterpret_cast<const ulonglong2*>(qh + 64);
          const ulonglong2 qd = *reinterpret_cast<const ulonglong2*>(qh + 96);
          unsigned long long s0 = mul2(qa.x, y1[0]), s1 = mul2(qc.x, y2[0]);
          fma2(s0, qa.y, y1[1]);
          fma2(s1, qc.y, y2[1]);
          fma2(s0, qe.x, y1[2]);
          fma2(s1, qd.x, y2[2]);
          fma2(s0, qe.y, y1[3]);
          fma2(s1, qd.y, y2[3]);
          sacc[h] = add2(s0, s1);
        }
      }
      float sv[G];
#pragma unroll
      for (int h = 0; h < G; ++h) sv[h] = lo2(sacc[h]) + hi2(sacc[h]);
      const int h0 = reduce_scatter8<G>(sv, part);
      constexpr int NV = G >= 8 ? G / 8 : 1;       // sums held per lane
      constexpr int DUP = G >= 8 ? 1 : 8 / G;      // lanes holding the same sums
      if (part % DUP == 0) {
#pragma unroll
        for (int i = 0; i < NV; ++i) scb[(h0 + i) * kScStride + r] = r < n_valid ? sv[i] : -INFINITY;
      }
    }
    __syncthreads();  // (A) scores ready; stage (j-1) % kDStages is free
    if (*abort_flag) break;
    if (tid == 0 && issued < nt) issue(issued++);

    // ---- softmax: warp w < NH owns heads w, w + NH, ...
    unsigned long long* ppb = pp + (j & 1) * kDKeys * G;
    float* alb = al + (j & 1) * G;
    if (warp < NH) {
#pragma unroll
      for (int a = 0; a < HPW; ++a) {
        const int h = warp + a * NH;
        const float s0 = scb[h * kScStride + lane], s1 = scb[h * kScStride + lane + 32];
        float mt = fmaxf(s0, s1);
#pragma unroll
        for (int o = 16; o; o >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, o));
        const float m_new = fmaxf(m_run[a], mt);
        float alpha = 1.f, p0 = 0.f, p1 = 0.f;
        if (m_new != -INFINITY) {  // warp-uniform
          alpha = ex2f(m_run[a] - m_new);
          p0 = ex2f(s0 - m_new);
          p1 = ex2f(s1 - m_new);
        }
        float ps = p0 + p1;
#pragma unroll
        for (int o = 16; o; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
        l_run[a] = l_run[a] * alpha + ps;
        m_run[a] = m_new;
        ppb[lane * G + h] = pk2(p0, p0);
        ppb[(lane + 32) * G + h] = pk2(p1, p1);
        if (lane == 0) alb[h] = alpha;
      }
    }
    if (j + 1 < nt) make_qt(j + 1);  // other buffer; read by Q K of tile j + 1
    __syncthreads();  // (B) p and alpha ready

    // ---- P V: warp w takes keys w + 8 m; lane owns dims 4 lane .. 4 lane + 3
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float a = alb[h];
      const unsigned long long a2 = pk2(a, a);
      acc[h][0] = mul2(acc[h][0], a2);
      acc[h][1] = mul2(acc[h][1], a2);
    }
#pragma unroll 2
    for (int kk = warp; kk < n_valid; kk += kDWarps) {
      const uint2 w = *reinterpret_cast<const uint2*>(vt + kk * kDRowB + lane * 8);
      const unsigned long long v01 = bf2_to_f2(w.x), v23 = bf2_to_f2(w.y);
      unsigned long long p2[G];
      if constexpr (G == 1) {
        p2[0] = ppb[kk];
      } else {
#pragma unroll
        for (int h = 0; h < G; h += 2) {
          const ulonglong2 t = *reinterpret_cast<const ulonglong2*>(ppb + kk * G + h);
          p2[h] = t.x;
          p2[h + 1] = t.y;
        }
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        fma2(acc[h][0], p2[h], v01);
        fma2(acc[h][1], p2[h], v23);
      }
    }
  }

  // every load issued must land before the ring is reused or the CTA exits
  if (tid == 0)
    for (int v = issued > kDStages ? issued - kDStages : 0; v < issued; ++v)
      tc::mbar_wait(&full[v % kDStages], (v / kDStages) & 1);
  if (warp < NH && lane == 0) {
#pragma unroll
    for (int a = 0; a < HPW; ++a) mlw[warp + a * NH] = make_float2(m_run[a], l_run[a]);
  }
  __syncthreads();
  float* red = reinterpret_cast<float*>(ring);  // [warp][G][D]
#pragma unroll
  for (int h = 0; h < G; ++h)
    *reinterpret_cast<float4*>(red + ((size_t)warp * G + h) * kDD + lane * 4) =
        make_float4(lo2(acc[h][0]), hi2(acc[h][0]), lo2(acc[h][1]), hi2(acc[h][1]));
  __syncthreads();
  for (int e = tid; e < G * kDD; e += kDThreads) {
    float o = 0.f;
#pragma unroll
    for (int w = 0; w < kDWarps; ++w) o += red[(size_t)w * G * kDD + e];
    const int h = e / kDD, d = e % kDD;
    const int64_t row_id = (int64_t)b * Hq + g * G + h;  // T == 1
    const float2 ml = mlw[h];
    if (n_split == 1) {
      const float inv = ml.y > 0.f ? 1.f / ml.y : 0.f;
      out[row_id * kDD + d] = __float2bfloat16(o * inv);
    } else {
      part_o[(row_id * n_split + split) * kDD + d] = o;
      if (d == 0) part_ml[row_id * n_split + split] = ml;
    }
  }
}

struct DecPlan {
  int n_split;
  size_t po_bytes, ml_bytes, total;
};

// Key splits: enough CTAs for about four waves of two resident CTAs per SM,
// each split keeping at least four 64-key tiles.
DecPlan dec_plan(int B, int Hq, int H, int D, int T_loc, int m_cap) {
  DecPlan p{};
  const int64_t base = (int64_t)B * H;
  const int64_t tiles = ((int64_t)m_cap + kDKeys - 1) / kDKeys + (T_loc + kDKeys - 1) / kDKeys;
  int64_t ns = (8LL * num_sms() + base - 1) / base;
  ns = std::min<int64_t>(ns, std::max<int64_t>(1, tiles / 4));
  ns = std::min<int64_t>(ns, 64);
  p.n_split = (int)std::max<int64_t>(ns, 1);
  const size_t rows = (size_t)B * Hq;
  p.po_bytes = p.n_split > 1 ? round_up(rows * p.n_split * D * sizeof(float), 256) : 0;
  p.ml_bytes = p.n_split > 1 ? round_up(rows * p.n_split * sizeof(float2), 256) : 0;
  p.total = p.po_bytes + p.ml_bytes;
  return p;
}

template <int G>
int launch_dec(int B, int T_loc, int Hq, int H, const void* q, const void* k_mem,
               const void* v_mem, const int32_t* mem_len, int m_cap, const void* k_loc,
               const void* v_loc, int pos0, float rope_base, float qscale, void* out, void* ws,
               cudaStream_t s) {
  const DecPlan p = dec_plan(B, Hq, H, kDD, T_loc, m_cap);
  unsigned char* w = static_cast<unsigned char*>(ws);
  float* part_o = reinterpret_cast<float*>(w);
  float2* part_ml = reinterpret_cast<float2*>(w + p.po_bytes);
  CUtensorMap tkm, tvm, tkl, tvl;
  const bool has_mem = m_cap > 0;
  const int64_t mem_rows = has_mem ? (int64_t)B * m_cap : (int64_t)B * T_loc;
  if (!tma_map_rows_bf16(&tkm, has_mem ? k_mem : k_loc, kDD, H, mem_rows, kDKeys) ||
      !tma_map_rows_bf16(&tvm, has_mem ? v_mem : v_loc, kDD, H, mem_rows, kDKeys) ||
      !tma_map_rows_bf16(&tkl, k_loc, kDD, H, (int64_t)B * T_loc, kDKeys) ||
      !tma_map_rows_bf16(&tvl, v_loc, kDD, H, (int64_t)B * T_loc, kDKeys))
    return note_cuda(cudaErrorInvalidValue);
  auto kern = attn_decode_kernel<G>;
  const size_t smem = DSmem<G>::ALLOC;
  int rc = ensure_smem_attr(reinterpret_cast<const void*>(kern), (int)smem);
  if (rc) return rc;
  const dim3 grid((unsigned)p.n_split, (unsigned)(B * H));
  kern<<<grid, kDThreads, smem, s>>>(tkm, tvm, tkl, tvl, T_loc, Hq, H,
                                     static_cast<const __nv_bfloat16*>(q), mem_len, m_cap, pos0,
                                     (double)rope_base, qscale, p.n_split,
                                     static_cast<__nv_bfloat16*>(out), part_o, part_ml,
                                     device_status_ptr());
  rc = check_launch();
  if (rc || p.n_split == 1) return rc;
  return attn_combine_bf16(B, 1, Hq, kDD, p.n_split, part_o, part_ml, out, s);
}

}  // namespace

bool attn_decode_supported(int T, int Hq, int H, int D) {
  if (T != 1 || D != kDD || H <= 0 || Hq % H) return false;
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
  if (!aligned16(k_loc) || !aligned16(v_loc) ||
      (m_cap > 0 && (!aligned16(k_mem) || !aligned16(v_mem))))
    return MSA_ERR_INVALID_ARG;
  if ((int64_t)B * H > 65535 || (int64_t)B * std::max(m_cap, T_loc) > INT32_MAX)
    return MSA_ERR_UNSUPPORTED;
  const int G = Hq / H;
#define MSA_DEC_CASE(GG)                                                                        \
  if (D == kDD && G == GG)                                                                      \
    return launch_dec<GG>(B, T_loc, Hq, H, q, k_mem, v_mem, mem_len, m_cap, k_loc, v_loc, pos0, \
                          rope_base, qscale, out, ws, s);
  MSA_DEC_CASE(1) MSA_DEC_CASE(2) MSA_DEC_CASE(4) MSA_DEC_CASE(8) MSA_DEC_CASE(16)
#undef MSA_DEC_CASE
  return MSA_ERR_UNSUPPORTED;
}

}  // namespace msa
