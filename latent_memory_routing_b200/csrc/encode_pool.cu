// Memory encoding: document-wise RoPE on token K fused with 64-token chunk
// means of K, V and K_r.
//
// Method: "EverMind-AI/MSA: routing top-k compressed documents inside
// attention ..." (hysenlabs.com), §"Document-wise RoPE resets every document
// to position zero" and §"Memory must be encoded offline before a query can
// reach it"; "深度分析MSA:把超长文档组织成可检索内部记忆的工程路径",
// §"三、文档如何变成 memory" / "2. chunk 压缩" (64 tokens per chunk,
// K -> K̄, V -> V̄, K_r -> K̄_r by mean pooling, 180 tokens -> 3 chunks).
//
// Design (HBM-bound stream).  encode_tma_kernel (the default): persistent
// CTAs, one per SM, each owning a contiguous range of chunks.  Producer
// threads stream, per (chunk, layer), the chunk's contiguous token rows with
// 1-D bulk copies (cp.async.bulk, 16 KB stages) into one ring per stream, so
// that each ring has one consumer group and a group never waits on a slot
// another group's stage may still hold -- the copy engine keeps 192 KB in
// flight per SM without a load instruction per 16 bytes.  The streams are K,
// V and K_r, except that in bf16 with two or more layers K -- whose consumers
// also rotate -- is split into two streams by layer parity, each with its
// own consumer group.  A consumer group's threads each own one 16-byte
// vector of a head and its rotate-half partner, add every row of their
// tensor from shared memory into fp32 registers (K rotated by the token's
// document-wise position from the chunk's (cos, sin) table, laid out so that
// a head's threads read consecutive words) and write the chunk's mean row
// once, so no partial sums cross threads.
// encode_pool_kernel (MSA_ENCODE_TMA=0): one CTA per chunk, looping over the
// L layers so the chunk's RoPE table is built once.  Each thread owns two 16-byte vectors
// of one head -- elements [v*VEC, v*VEC+VEC) and the rotate-half partners at
// +D/2 -- so the rotation needs no data exchange; R token rows are in flight
// per CTA.  Loads are 16-byte, coalesced and L1-bypassing; sums are fp32;
// the R partial sums are combined through shared memory and each output row
// is written once with 16-byte stores.
#include <algorithm>
#include <cstdlib>

#include "msa_common.cuh"
#include "tc_ptx.cuh"

namespace msa {
namespace {

constexpr int kEncThreads = 256;
constexpr int kMaxChunk = 64;

template <typename T, int D>
__global__ void __launch_bounds__(kEncThreads)
encode_pool_kernel(int L, int64_t n_tok, int n_docs, int H, int R,
                   const T* __restrict__ k_tok, const T* __restrict__ v_tok,
                   const T* __restrict__ kr_tok,
                   const int64_t* __restrict__ tok_off,
                   const int64_t* __restrict__ chunk_off, int64_t n_chunks,
                   double base, int chunk, T* __restrict__ k_bar,
                   T* __restrict__ v_bar, T* __restrict__ kr_bar) {
  constexpr int VEC = Vec16<T>::N;
  constexpr int HALF = D / 2;
  constexpr int UPH = HALF / VEC;  // pair-vectors per head
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float2* cs_tab = reinterpret_cast<float2*>(smem_raw);           // [64][HALF]
  float* red = reinterpret_cast<float*>(cs_tab + kMaxChunk * HALF);  // [R][3][H*D]
  __shared__ double w_tab[HALF];
  __shared__ int64_t s_tok0, s_p0;
  __shared__ int s_rows;

  const int tid = threadIdx.x;
  const int U = H * UPH;
  const int u = tid % U, r = tid / U;
  const int h = u / UPH, v = u % UPH;
  const int64_t c = blockIdx.x;
  const int64_t row_elems = (int64_t)H * D;

  if (tid < 32) {
    const int64_t d = warp_find_segment(chunk_off, n_docs, c);
    if (tid == 0) {
      const int64_t j = c - chunk_off[d];
      const int64_t t0 = tok_off[d] + j * chunk;
      const int64_t left = tok_off[d + 1] - t0;
      s_tok0 = t0;
      s_p0 = j * chunk;  // position of the chunk's first token in its doc
      s_rows = (int)(left < 0 ? 0 : (left < chunk ? left : chunk));
    }
  }
  for (int i = tid; i < HALF; i += blockDim.x) w_tab[i] = rope_inv_freq(base, i, D);
  __syncthreads();
  const int rows = s_rows;
  const int64_t tok0 = s_tok0, p0 = s_p0;
  for (int e = tid; e < rows * HALF; e += blockDim.x) {
    const int t = e / HALF, i = e - (e / HALF) * HALF;
    cs_tab[e] = rope_cs(p0 + t, w_tab[i]);
  }
  __syncthreads();

  const float inv_n = rows > 0 ? 1.0f / (float)rows : 0.f;
  const int64_t col_lo = (int64_t)h * D + v * VEC;
  for (int l = 0; l < L; ++l) {
    float ak[2][VEC], av[2][VEC], ar[2][VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
      ak[0][e] = ak[1][e] = av[0][e] = av[1][e] = ar[0][e] = ar[1][e] = 0.f;
    }
    if (r < R) {
      const int64_t layer_row0 = (int64_t)l * n_tok + tok0;
#pragma unroll 2
      for (int t = r; t < rows; t += R) {
        const int64_t off = (layer_row0 + t) * row_elems + col_lo;
        const uint4 k0 = ld_stream16(k_tok + off), k1 = ld_stream16(k_tok + off + HALF);
        const uint4 v0 = ld_stream16(v_tok + off), v1 = ld_stream16(v_tok + off + HALF);
        const uint4 r0 = ld_stream16(kr_tok + off), r1 = ld_stream16(kr_tok + off + HALF);
        float x1[VEC], x2[VEC], f[VEC];
        Vec16<T>::unpack(k0, x1);
        Vec16<T>::unpack(k1, x2);
        const float2* cs = cs_tab + t * HALF + v * VEC;
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
          const float2 q = cs[e];
          ak[0][e] += x1[e] * q.x - x2[e] * q.y;
          ak[1][e] += x2[e] * q.x + x1[e] * q.y;
        }
        Vec16<T>::unpack(v0, f);
#pragma unroll
        for (int e = 0; e < VEC; ++e) av[0][e] += f[e];
        Vec16<T>::unpack(v1, f);
#pragma unroll
        for (int e = 0; e < VEC; ++e) av[1][e] += f[e];
        Vec16<T>::unpack(r0, f);
#pragma unroll
        for (int e = 0; e < VEC; ++e) ar[0][e] += f[e];
        Vec16<T>::unpack(r1, f);
#pragma unroll
        for (int e = 0; e < VEC; ++e) ar[1][e] += f[e];
      }
      float* my = red + (int64_t)r * 3 * row_elems;
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        my[col_lo + e] = ak[0][e];
        my[col_lo + HALF + e] = ak[1][e];
        my[row_elems + col_lo + e] = av[0][e];
        my[row_elems + col_lo + HALF + e] = av[1][e];
        my[2 * row_elems + col_lo + e] = ar[0][e];
        my[2 * row_elems + col_lo + HALF + e] = ar[1][e];
      }
    }
    __syncthreads();
    const int64_t out_row = ((int64_t)l * n_chunks + c) * row_elems;
    for (int64_t e0 = (int64_t)tid * VEC; e0 < 3 * row_elems;
         e0 += (int64_t)blockDim.x * VEC) {
      const int tensor = (int)(e0 / row_elems);
      const int64_t col = e0 - tensor * row_elems;
      float o[VEC];
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        float s = 0.f;
        for (int rr = 0; rr < R; ++rr) s += red[(int64_t)rr * 3 * row_elems + e0 + e];
        o[e] = s * inv_n;
      }
      T* dst = tensor == 0 ? k_bar : (tensor == 1 ? v_bar : kr_bar);
      st16(dst + out_row + col, Vec16<T>::pack(o));
    }
    __syncthreads();
  }
}

constexpr int kEncStage = 16384;  // bytes per ring stage
constexpr int kEncStages = 4;     // stages per tensor stream: one ring per consumer group
constexpr int kEncRing = 3 * kEncStages;  // stages in all rings

// Streams: in bf16 with L >= 2 layers, K -- whose consumers also rotate, the
// slowest of the three -- is split into two streams by layer parity, each
// with its own ring of kEncStages / 2 stages and its own consumer group, so
// twice the threads work on K and no partial sums have to be combined; V
// and K_r keep one stream of kEncStages stages each.  Otherwise (one layer,
// or fp32, whose four groups would not fit a CTA's threads) the three
// tensors are one stream each.
struct EncStreams {
  bool split;
  __host__ __device__ int count() const { return split ? 4 : 3; }
  __host__ __device__ int tensor(int s) const { return split ? (s < 2 ? 0 : s - 1) : s; }
  __host__ __device__ int stages(int s) const {
    return split && s < 2 ? kEncStages / 2 : kEncStages;
  }
  __host__ __device__ int first_stage(int s) const {
    return split ? (s < 2 ? s * (kEncStages / 2) : (s - 1) * kEncStages) : s * kEncStages;
  }
  // stream s carries layer l of its tensor
  __host__ __device__ bool carries(int s, int l) const { return !split || s >= 2 || (l & 1) == s; }
};

// Threads: one producer warp + three or four consumer groups of Ug (U
// rounded up to a warp) threads, U = H * (D/2) / VEC.
template <typename T, int D>
constexpr int enc_tma_max_threads() {
  return 32 + (sizeof(T) == 2 ? 4 : 3) * (16 * (D / 2) / Vec16<T>::N);
}

template <typename T, int D>
__global__ void __launch_bounds__(enc_tma_max_threads<T, D>(), 1)
encode_tma_kernel(int L, int64_t n_tok, int n_docs, int H, int U, int Ug, int RS, int split_k,
                  const T* __restrict__ k_tok, const T* __restrict__ v_tok,
                  const T* __restrict__ kr_tok, const int64_t* __restrict__ tok_off,
                  const int64_t* __restrict__ chunk_off, int64_t n_chunks, double base,
                  int chunk, T* __restrict__ k_bar, T* __restrict__ v_bar,
                  T* __restrict__ kr_bar, T* __restrict__ kr_hat, int* status) {
  constexpr int VEC = Vec16<T>::N;
  constexpr int HALF = D / 2;
  constexpr int UPH = HALF / VEC;
  extern __shared__ __align__(1024) unsigned char enc_dsm[];
  unsigned char* ring = tc::smem_align<1024>(enc_dsm);
  // ring of stream s: stages [first_stage(s), first_stage(s) + stages(s))
  float2* cs_tab = reinterpret_cast<float2*>(ring + kEncRing * kEncStage);  // [64][HALF]
  __shared__ uint64_t full[kEncRing], empty[kEncRing];
  const EncStreams S{split_k != 0};
  __shared__ double w_tab[HALF];
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row_elems = (int64_t)H * D;
  const uint32_t row_bytes = (uint32_t)(row_elems * sizeof(T));
  const int64_t cb = (int64_t)blockIdx.x * n_chunks / gridDim.x;
  const int64_t ce = (int64_t)(blockIdx.x + 1) * n_chunks / gridDim.x;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kEncRing; ++i) {
      tc::mbar_init(&full[i], 1);
      tc::mbar_init(&empty[i], Ug / 32);
    }
    abort_flag = 0;
    tc::fence_mbar_init();
  }
  for (int i = threadIdx.x; i < HALF; i += blockDim.x) w_tab[i] = rope_inv_freq(base, i, D);
  __syncthreads();
  volatile int* abort_v = &abort_flag;
  auto wait = [&](uint64_t* bar, uint32_t parity) {
    if (*abort_v) return;
    if (!tc::mbar_wait(bar, parity)) {
      record_error(status, MSA_ERR_TIMEOUT);
      *abort_v = 1;
    }
  };
  // the chunk's document: a bisection for the first chunk, then a forward
  // walk (a CTA's chunks are consecutive), with the document's offsets kept
  // in registers so that most chunks need no global load
  int64_t d = 0;
  {
    int64_t lo = 0, hi = n_docs;
    while (hi - lo > 1) {
      const int64_t mid = (lo + hi) >> 1;
      if (__ldg(chunk_off + mid) <= cb) lo = mid; else hi = mid;
    }
    d = lo;
  }
  int64_t c_lo = __ldg(chunk_off + d), c_hi = __ldg(chunk_off + d + 1);
  int64_t t_lo = __ldg(tok_off + d), t_hi = __ldg(tok_off + d + 1);
  auto locate = [&](int64_t c, int64_t& tok0, int& rows, int64_t& p0) {
    while (c >= c_hi && d + 1 < n_docs) {
      ++d;
      c_lo = c_hi;
      c_hi = __ldg(chunk_off + d + 1);
      t_lo = t_hi;
      t_hi = __ldg(tok_off + d + 1);
    }
    const int64_t j = c - c_lo;
    tok0 = t_lo + j * chunk;
    const int64_t left = t_hi - tok0;
    rows = (int)(left < 0 ? 0 : (left < chunk ? left : chunk));
    p0 = j * chunk;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // lane s streams stream s into its own ring, so that no ring waits
    // behind another's slot
    if (lane < S.count()) {
      const int sidx = lane, t = S.tensor(sidx);
      const int ns = S.stages(sidx), s0 = S.first_stage(sidx);
      const T* src = t == 0 ? k_tok : (t == 1 ? v_tok : kr_tok);
      uint32_t u = 0;  // stages issued to this stream's ring
      for (int64_t c = cb; c < ce; ++c) {
        int64_t tok0, p0;
        int rows;
        locate(c, tok0, rows, p0);
        const int nstg = (rows + RS - 1) / RS;
        for (int l = 0; l < L; ++l) {
          if (!S.carries(sidx, l)) continue;
          for (int g = 0; g < nstg; ++g, ++u) {
            const int st = s0 + (int)(u % ns);
            wait(&empty[st], ((u / ns) & 1) ^ 1);
            if (*abort_v) continue;
            const int nr = min(RS, rows - g * RS);
            tc::mbar_arrive_expect_tx(&full[st], (uint32_t)nr * row_bytes);
            tc::bulk_load(ring + (size_t)st * kEncStage,
                          src + ((int64_t)l * n_tok + tok0 + (int64_t)g * RS) * row_elems,
                          (uint32_t)nr * row_bytes, &full[st]);
          }
        }
      }
      // every copy issued must land before the CTA exits
      for (uint32_t v = u > (uint32_t)ns ? u - ns : 0; v < u; ++v)
        tc::mbar_wait(&full[s0 + v % ns], (v / ns) & 1);
    }
  } else {
    // ----------------------------------------------------------- consumers
    const int sidx = (warp - 1) / (Ug / 32);         // the group's stream
    const int t = S.tensor(sidx);                    // 0: K, 1: V, 2: K_r
    const int ns = S.stages(sidx), s0 = S.first_stage(sidx);
    const int jt = (int)threadIdx.x - 32 - sidx * Ug;  // index in the group
    const int nk = S.split ? 2 : 1;                  // groups working on K
    const int jk = jt + (t == 0 && S.split ? sidx : 0) * Ug;  // index among them
    const bool active = jt < U;
    const int h = jt / UPH, v = jt % UPH;
    const int64_t col_lo = (int64_t)h * D + v * VEC;
    T* dst = t == 0 ? k_bar : (t == 1 ? v_bar : kr_bar);
    uint32_t u = 0;
    for (int64_t c = cb; c < ce; ++c) {
      int64_t tok0, p0;
      int rows;
      locate(c, tok0, rows, p0);
      const int nstg = (rows + RS - 1) / RS;
      if (t == 0) {  // the K groups rebuild the chunk's (cos, sin) table
        asm volatile("bar.sync 1, %0;" ::"r"(nk * Ug) : "memory");  // old table no longer read
        // frequency i: an exact anchor at p0 (angle reduced in double), then
        // one rotation by w_i per row, in double
        // stored transposed within a row, [row][e][v] for frequency
        // i = v * VEC + e, so that the threads of a head (consecutive v)
        // read consecutive 8-byte words: no bank conflicts (read in the
        // row's order [v * VEC + e], neighbouring threads' words sit 64 B
        // apart and four of a head's eight threads share a bank)
        for (int i = jk; i < HALF; i += nk * Ug) {
          const double w = w_tab[i];
          double sa, ca, sw, cw;
          const double two_pi = 6.283185307179586;
          const double th = (double)p0 * w;
          sincos(fma(-rint(th * (1.0 / two_pi)), two_pi, th), &sa, &ca);
          sincos(w, &sw, &cw);
          const int slot = (i % VEC) * UPH + i / VEC;
          for (int r = 0; r < rows; ++r) {
            cs_tab[r * HALF + slot] = make_float2((float)ca, (float)sa);
            const double cn = ca * cw - sa * sw;
            sa = sa * cw + ca * sw;
            ca = cn;
          }
        }
        asm volatile("bar.sync 1, %0;" ::"r"(nk * Ug) : "memory");
      }
      const float inv_n = rows > 0 ? 1.0f / (float)rows : 0.f;
      for (int l = 0; l < L; ++l) {
        if (!S.carries(sidx, l)) continue;
        float a1[VEC], a2[VEC];
#pragma unroll
        for (int e = 0; e < VEC; ++e) a1[e] = a2[e] = 0.f;
        for (int g = 0; g < nstg; ++g, ++u) {
          const int st = s0 + (int)(u % ns);
          wait(&full[st], (u / ns) & 1);
          const int nr = min(RS, rows - g * RS);
          if (active && !*abort_v) {
            const unsigned char* base_row = ring + (size_t)st * kEncStage;
#pragma unroll 2
            for (int rr = 0; rr < nr; ++rr) {
              const unsigned char* row = base_row + (size_t)rr * row_bytes;
              const uint4 q1 = *reinterpret_cast<const uint4*>(row + col_lo * sizeof(T));
              const uint4 q2 =
                  *reinterpret_cast<const uint4*>(row + (col_lo + HALF) * sizeof(T));
              float x1[VEC], x2[VEC];
              Vec16<T>::unpack(q1, x1);
              Vec16<T>::unpack(q2, x2);
              if (t == 0) {
                const float2* cs = cs_tab + (g * RS + rr) * HALF + v;
#pragma unroll
                for (int e = 0; e < VEC; ++e) {
                  const float2 q = cs[e * UPH];
                  a1[e] += x1[e] * q.x - x2[e] * q.y;
                  a2[e] += x2[e] * q.x + x1[e] * q.y;
                }
              } else {
#pragma unroll
                for (int e = 0; e < VEC; ++e) {
                  a1[e] += x1[e];
                  a2[e] += x2[e];
                }
              }
            }
          }
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(&empty[st]);
        }
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
          a1[e] *= inv_n;
          a2[e] *= inv_n;
        }
        const uint4 p1 = Vec16<T>::pack(a1), p2 = Vec16<T>::pack(a2);
        const int64_t o_off = ((int64_t)l * n_chunks + c) * row_elems + col_lo;
        if (active && dst) {
          st16(dst + o_off, p1);
          st16(dst + o_off + HALF, p2);
        }
        if (t == 2 && kr_hat) {
          // the prepared routing row: the (chunk, head) row of K̄_r as
          // rounded above, divided by max(|row|, 1e-12) and rounded again --
          // the arithmetic of the bank preparation step in the same order
          // (fp32 squares of each 8-element piece, the pieces v and v + UPH
          // of this thread added, then a butterfly over the head's UPH
          // threads, which sit on consecutive lanes), so the bytes are those
          // msa_route_prepare_bank writes from K̄_r.  Whole warps take part
          // in the shuffles (an inactive lane holds zeros in its own head
          // group).
          float f1[VEC], f2[VEC];
          Vec16<T>::unpack(p1, f1);
          Vec16<T>::unpack(p2, f2);
          float s1 = 0.f, s2 = 0.f;
#pragma unroll
          for (int e = 0; e < VEC; ++e) {
            s1 = fmaf(f1[e], f1[e], s1);
            s2 = fmaf(f2[e], f2[e], s2);
          }
          float ss = s1 + s2;
#pragma unroll
          for (int o = UPH / 2; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
          const float inv = 1.0f / fmaxf(sqrtf(ss), 1e-12f);
#pragma unroll
          for (int e = 0; e < VEC; ++e) {
            f1[e] *= inv;
            f2[e] *= inv;
          }
          if (active) {
            st16(kr_hat + o_off, Vec16<T>::pack(f1));
            st16(kr_hat + o_off + HALF, Vec16<T>::pack(f2));
          }
        }
      }
    }
  }
}

bool encode_tma_enabled() {
  static const bool on = [] {
    const char* e = getenv("MSA_ENCODE_TMA");
    return !(e && e[0] == '0');
  }();
  return on;
}

__global__ void chunk_offsets_kernel(int n_docs, const int64_t* __restrict__ tok_off,
                                     int chunk, int64_t* __restrict__ chunk_off,
                                     int* status) {
  __shared__ int64_t part[1024];
  const int tid = threadIdx.x;
  const int per = (n_docs + blockDim.x - 1) / blockDim.x;
  const int d0 = tid * per;
  const int d1 = min(d0 + per, n_docs);
  int64_t s = 0;
  for (int d = d0; d < d1; ++d) {
    const int64_t len = tok_off[d + 1] - tok_off[d];
    if (len <= 0) record_error(status, MSA_ERR_INVALID_ARG);
    else s += (len + chunk - 1) / chunk;
  }
  part[tid] = s;
  __syncthreads();
  for (int off = 1; off < (int)blockDim.x; off <<= 1) {  // inclusive scan
    const int64_t add = tid >= off ? part[tid - off] : 0;
    __syncthreads();
    part[tid] += add;
    __syncthreads();
  }
  int64_t run = part[tid] - s;  // exclusive
  if (tid == 0) chunk_off[0] = 0;
  for (int d = d0; d < d1; ++d) {
    const int64_t len = tok_off[d + 1] - tok_off[d];
    if (len > 0) run += (len + chunk - 1) / chunk;
    chunk_off[d + 1] = run;
  }
}

// rh (the prepared routing bank) != nullptr: bf16 only, and always on the
// bulk-copy kernel.
template <typename T, int D>
int launch_encode(int L, int64_t n_tok, int n_docs, int H, const void* k,
                  const void* v, const void* kr, const int64_t* toff,
                  const int64_t* coff, int64_t n_chunks, float base, int chunk,
                  void* kb, void* vb, void* rb, void* rh, cudaStream_t s) {
  constexpr int VEC = Vec16<T>::N;
  const int64_t row_bytes = (int64_t)H * D * (int64_t)sizeof(T);
  if ((encode_tma_enabled() || rh) && row_bytes % 16 == 0 && row_bytes <= kEncStage) {
    const int U = H * (D / 2 / VEC);
    const int Ug = (U + 31) / 32 * 32;
    const int RS = (int)std::min<int64_t>(chunk, kEncStage / row_bytes);
    const size_t smem =
        1024 + (size_t)kEncRing * kEncStage + sizeof(float2) * kMaxChunk * (D / 2);
    auto kern = encode_tma_kernel<T, D>;
    int rc = ensure_smem_attr(reinterpret_cast<const void*>(kern), (int)smem);
    if (rc) return rc;
    if (n_chunks == 0) return MSA_OK;
    const int grid = (int)std::min<int64_t>(n_chunks, num_sms());
    const bool split = sizeof(T) == 2 && L >= 2;
    kern<<<grid, 32 + EncStreams{split}.count() * Ug, smem, s>>>(
        L, n_tok, n_docs, H, U, Ug, RS, split ? 1 : 0, static_cast<const T*>(k), static_cast<const T*>(v),
        static_cast<const T*>(kr), toff, coff, n_chunks, (double)base, chunk,
        static_cast<T*>(kb), static_cast<T*>(vb), static_cast<T*>(rb), static_cast<T*>(rh),
        device_status_ptr());
    return check_launch();
  }
  if (rh) return MSA_ERR_UNSUPPORTED;
  const int U = H * (D / 2 / VEC);
  const int R = U >= kEncThreads ? 1 : kEncThreads / U;
  const int threads = U * R;
  if (threads > kEncThreads) return MSA_ERR_UNSUPPORTED;
  const size_t smem = sizeof(float2) * kMaxChunk * (D / 2) +
                      sizeof(float) * (size_t)R * 3 * H * D;
  auto kern = encode_pool_kernel<T, D>;
  int rc = ensure_smem_attr(reinterpret_cast<const void*>(kern), (int)smem);
  if (rc) return rc;
  if (n_chunks == 0) return MSA_OK;
  kern<<<(unsigned)n_chunks, threads, smem, s>>>(
      L, n_tok, n_docs, H, R, static_cast<const T*>(k), static_cast<const T*>(v),
      static_cast<const T*>(kr), toff, coff, n_chunks, (double)base, chunk,
      static_cast<T*>(kb), static_cast<T*>(vb), static_cast<T*>(rb));
  return check_launch();
}

}  // namespace
}  // namespace msa

extern "C" int msa_chunk_offsets(int n_docs, const int64_t* tok_offsets,
                                 int chunk, int64_t* chunk_offsets,
                                 msa_stream_t stream) {
  if (n_docs <= 0 || !tok_offsets || !chunk_offsets) return MSA_ERR_INVALID_ARG;
  if (chunk < 1 || chunk > msa::kMaxChunk) return MSA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (int rc = msa::debug_check_offsets(tok_offsets, n_docs, INT64_MAX, s)) return rc;
  msa::chunk_offsets_kernel<<<1, 1024, 0, s>>>(n_docs, tok_offsets, chunk,
                                               chunk_offsets,
                                               msa::device_status_ptr());
  return msa::debug_finish(msa::check_launch(), s);
}

namespace msa {
namespace {

int encode_pool_impl(msa_dtype dt, int L, int64_t n_tok, int n_docs, int H, int D,
                     const void* k_tok, const void* v_tok, const void* kr_tok,
                     const int64_t* tok_offsets, const int64_t* chunk_offsets, int64_t n_chunks,
                     float rope_base, int chunk, void* k_bar, void* v_bar, void* kr_bar,
                     void* kr_hat, cudaStream_t s) {
  if (L <= 0 || n_tok <= 0 || n_docs <= 0 || n_chunks < 0 || H <= 0) return MSA_ERR_INVALID_ARG;
  if (!k_tok || !v_tok || !kr_tok || !tok_offsets || !chunk_offsets || !k_bar || !v_bar ||
      (!kr_bar && !kr_hat))
    return MSA_ERR_INVALID_ARG;
  if (!aligned16(k_tok) || !aligned16(v_tok) || !aligned16(kr_tok) || !aligned16(k_bar) ||
      !aligned16(v_bar) || !aligned16(kr_bar) || !aligned16(kr_hat))
    return MSA_ERR_INVALID_ARG;
  if (chunk < 1 || chunk > kMaxChunk || !(rope_base > 0.f)) return MSA_ERR_INVALID_ARG;
  if (H < 1 || H > 16 || (D != 64 && D != 128)) return MSA_ERR_UNSUPPORTED;
  if (n_chunks > 0x7fffffffLL) return MSA_ERR_UNSUPPORTED;
  if (dt != MSA_F32 && dt != MSA_BF16) return MSA_ERR_INVALID_ARG;
  if (kr_hat && dt != MSA_BF16) return MSA_ERR_UNSUPPORTED;
  if (int rc = debug_check_offsets(tok_offsets, n_docs, n_tok, s)) return rc;
  if (int rc = debug_check_offsets(chunk_offsets, n_docs, n_chunks, s)) return rc;
  int rc;
  if (dt == MSA_F32)
    rc = D == 64 ? launch_encode<float, 64>(L, n_tok, n_docs, H, k_tok, v_tok, kr_tok,
                                            tok_offsets, chunk_offsets, n_chunks, rope_base,
                                            chunk, k_bar, v_bar, kr_bar, nullptr, s)
                 : launch_encode<float, 128>(L, n_tok, n_docs, H, k_tok, v_tok, kr_tok,
                                             tok_offsets, chunk_offsets, n_chunks, rope_base,
                                             chunk, k_bar, v_bar, kr_bar, nullptr, s);
  else
    rc = D == 64 ? launch_encode<__nv_bfloat16, 64>(L, n_tok, n_docs, H, k_tok, v_tok, kr_tok,
                                                    tok_offsets, chunk_offsets, n_chunks,
                                                    rope_base, chunk, k_bar, v_bar, kr_bar,
                                                    kr_hat, s)
                 : launch_encode<__nv_bfloat16, 128>(L, n_tok, n_docs, H, k_tok, v_tok, kr_tok,
                                                     tok_offsets, chunk_offsets, n_chunks,
                                                     rope_base, chunk, k_bar, v_bar, kr_bar,
                                                     kr_hat, s);
  return debug_finish(rc, s);
}

}  // namespace
}  // namespace msa

extern "C" int msa_encode_pool(msa_dtype dt, int L, int64_t n_tok, int n_docs,
                               int H, int D, const void* k_tok,
                               const void* v_tok, const void* kr_tok,
                               const int64_t* tok_offsets,
                               const int64_t* chunk_offsets, int64_t n_chunks,
                               float rope_base, int chunk, void* k_bar,
                               void* v_bar, void* kr_bar, msa_stream_t stream) {
  if (!kr_bar) return MSA_ERR_INVALID_ARG;
  return msa::encode_pool_impl(dt, L, n_tok, n_docs, H, D, k_tok, v_tok, kr_tok, tok_offsets,
                               chunk_offsets, n_chunks, rope_base, chunk, k_bar, v_bar, kr_bar,
                               nullptr, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int msa_encode_pool_prepared(msa_dtype dt, int L, int64_t n_tok, int n_docs, int H,
                                        int D, const void* k_tok, const void* v_tok,
                                        const void* kr_tok, const int64_t* tok_offsets,
                                        const int64_t* chunk_offsets, int64_t n_chunks,
                                        float rope_base, int chunk, void* k_bar, void* v_bar,
                                        void* kr_bar, void* kr_hat, msa_stream_t stream) {
  if (!kr_hat) return MSA_ERR_INVALID_ARG;
  return msa::encode_pool_impl(dt, L, n_tok, n_docs, H, D, k_tok, v_tok, kr_tok, tok_offsets,
                               chunk_offsets, n_chunks, rope_base, chunk, k_bar, v_bar, kr_bar,
                               kr_hat, reinterpret_cast<cudaStream_t>(stream));
}
