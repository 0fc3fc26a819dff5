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
//   * persistent CTAs, one per SM, walk 128-chunk tiles round-robin;
//   * warp 0 (one lane) TMA-loads, per (tile, head), the tile's K̄_r rows of
//     that head (128 x D bf16, 128B-swizzled) and the head's normalised
//     query columns (N x D) into a multi-stage shared-memory ring;
//   * warp 1 (one lane) issues tcgen05.mma M=128 (chunks) x N (query
//     columns) x K=D per head into one of two TMEM accumulators, so the
//     next head's MMAs overlap the epilogue of this one;
//   * warps 2..9 (the epilogue) compute |K̄_r[c,h]| from the same shared
//     tile, read the head's 128 x N scores from TMEM (one chunk row per
//     thread, half of the columns per warpgroup), and accumulate
//     inv|k| * score in registers -- the query side is pre-normalised with
//     1/H folded in, so after the last head the registers hold the
//     head-mean cosine;
//   * the tile's row values go back to TMEM once, are reduced over each
//     query's tokens (max), then over the rows of each document inside the
//     warp (segmented shuffle max), and only one order-preserving atomicMax
//     per (query, document segment) reaches global memory.
// Scores never round-trip through HBM.  No cluster multicast is used.
#include <cudaTypedefs.h>

#include <algorithm>

#include "msa_common.cuh"
#include "route_tc.cuh"
#include "tc_ptx.cuh"

namespace msa {
namespace {

constexpr int kTile = 128;  // chunks per tile = MMA M = TMEM lanes
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kWindow = 256;  // documents cached per tile for chunk -> doc
constexpr int kEpiBar = 1;    // named barrier of the epilogue warps

template <int N, int D>
struct Cfg {
  static constexpr int KB = D / 64;                   // 64-element K blocks
  static constexpr int A_BYTES = KB * kTile * 128;    // one head of a tile
  static constexpr int B_BYTES = KB * N * 128;        // one head of the queries
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int STAGES_FIT = (196 * 1024) / STAGE;
  static constexpr int STAGES = STAGES_FIT > 4 ? 4 : STAGES_FIT;
  static constexpr int TMEM_COLS = 2 * N < 32 ? 32 : 2 * N;
  static constexpr int HALF_N = N / 2;
  static constexpr uint32_t IDESC = tc::idesc_bf16_f32(kTile, N);
  static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE;
  static_assert(STAGES >= 2, "need a double-buffered ring");
  static_assert(N % 64 == 0 && N >= 64 && N <= 256, "N: whole 32-column TMEM loads per half");
};

struct Aux {
  uint64_t full[4], empty[4], accf[2], acce[2];
  uint32_t tmem_base;
  int abort_flag;
  int d0;
  int doc_row[kTile];
  float npart[2][2][kTile];
  int64_t win[kWindow + 1];
};

__device__ __forceinline__ void epi_bar() {
  asm volatile("bar.sync %0, %1;" ::"n"(kEpiBar), "n"(32 * kEpiWarps) : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]),
      "f"(v[8]), "f"(v[9]), "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]),
      "f"(v[15]), "f"(v[16]), "f"(v[17]), "f"(v[18]), "f"(v[19]), "f"(v[20]), "f"(v[21]),
      "f"(v[22]), "f"(v[23]), "f"(v[24]), "f"(v[25]), "f"(v[26]), "f"(v[27]), "f"(v[28]),
      "f"(v[29]), "f"(v[30]), "f"(v[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ float sumsq8(const uint4& v) {
  float a = bf16lo(v.x), b = bf16hi(v.x), c = bf16lo(v.y), d = bf16hi(v.y);
  float e = bf16lo(v.z), f = bf16hi(v.z), g = bf16lo(v.w), h = bf16hi(v.w);
  return a * a + b * b + c * c + d * d + e * e + f * f + g * g + h * h;
}

template <int N, int D>
__global__ void __launch_bounds__(kThreads, 1)
route_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
                int H, int NT, int T, int n_pass, int64_t C, int64_t n_tiles,
                const int64_t* __restrict__ coff, int n_docs, uint32_t* __restrict__ doc_u,
                uint32_t* __restrict__ chunk_u, int* __restrict__ status) {
  using K = Cfg<N, D>;
  extern __shared__ __align__(1024) unsigned char smem_dyn[];
  __shared__ Aux aux;
  unsigned char* ring = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < K::STAGES; ++i) {
      tc::mbar_init(&aux.full[i], 1);
      tc::mbar_init(&aux.empty[i], 1 + kEpiWarps);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&aux.accf[i], 1);
      tc::mbar_init(&aux.acce[i], kEpiWarps);
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
  volatile int* abort_flag = &aux.abort_flag;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tc::tma_prefetch_desc(&tm_k);
      tc::tma_prefetch_desc(&tm_q);
      uint32_t u = 0;
      for (int p = 0; p < n_pass && !*abort_flag; ++p)
        for (int64_t tile = blockIdx.x; tile < n_tiles && !*abort_flag; tile += gridDim.x)
          for (int h = 0; h < H; ++h, ++u) {
            const int st = u % K::STAGES;
            const uint32_t ph = (u / K::STAGES) & 1u;
            if (!tc::mbar_wait(&aux.empty[st], ph ^ 1u)) {
              record_error(status, MSA_ERR_TIMEOUT);
              *abort_flag = 1;
              break;
            }
            unsigned char* a = ring + st * K::STAGE;
            unsigned char* b = a + K::A_BYTES;
            tc::mbar_arrive_expect_tx(&aux.full[st], K::STAGE);
#pragma unroll
            for (int kb = 0; kb < K::KB; ++kb)
              tc::tma_load_3d(a + kb * kTile * 128, &tm_k, &aux.full[st], kb * 64, h,
                              (int32_t)(tile * kTile));
#pragma unroll
            for (int kb = 0; kb < K::KB; ++kb)
              tc::tma_load_3d(b + kb * N * 128, &tm_q, &aux.full[st], kb * 64, p * N, h);
          }
      // Drain: every load issued must have landed before the CTA exits.
      const uint32_t issued = u;
      for (uint32_t v = issued > (uint32_t)K::STAGES ? issued - K::STAGES : 0; v < issued; ++v)
        tc::mbar_wait(&aux.full[v % K::STAGES], (v / K::STAGES) & 1u);
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      uint32_t u = 0;
      for (int p = 0; p < n_pass && !*abort_flag; ++p)
        for (int64_t tile = blockIdx.x; tile < n_tiles && !*abort_flag; tile += gridDim.x)
          for (int h = 0; h < H; ++h, ++u) {
            const int st = u % K::STAGES;
            const uint32_t ph = (u / K::STAGES) & 1u;
            const int ab = u & 1;
            const uint32_t aph = (u >> 1) & 1u;
            if (!tc::mbar_wait(&aux.full[st], ph) || !tc::mbar_wait(&aux.acce[ab], aph ^ 1u)) {
              record_error(status, MSA_ERR_TIMEOUT);
              *abort_flag = 1;
              break;
            }
            tc::tc_fence_after();
            const uint32_t a0 = tc::smem_u32(ring + st * K::STAGE);
            const uint32_t b0 = a0 + K::A_BYTES;
            const uint32_t d_tmem = tmem + ab * N;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t koff = (kk & 3) * 32;  // 16 bf16 = 32 B inside the swizzle atom
              const uint64_t ad = tc::sdesc_kmajor_sw128(a0 + (kk >> 2) * (kTile * 128) + koff);
              const uint64_t bd = tc::sdesc_kmajor_sw128(b0 + (kk >> 2) * (N * 128) + koff);
              tc::mma_bf16_ss(d_tmem, ad, bd, K::IDESC, kk > 0 ? 1u : 0u);
            }
            tc::mma_commit(&aux.empty[st]);
            tc::mma_commit(&aux.accf[ab]);
          }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;
    const int quad = warp & 3;  // TMEM lane quarter this warp may access
    const int half = ew >> 2;   // which half of the query columns
    const int row = quad * 32 + lane;
    const int et = ew * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    float acc[K::HALF_N];
    uint32_t u = 0;
    for (int p = 0; p < n_pass; ++p) {
      const int col_begin = p * N + half * K::HALF_N;  // first global column of this half
      for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
        const int64_t c0 = tile * kTile;
        const int64_t c = c0 + row;
        // chunk -> document for the tile's rows
        if (ew == 0) {
          const int64_t d0 = warp_find_segment(coff, n_docs, c0);
          if (lane == 0) aux.d0 = (int)d0;
        }
        epi_bar();
        const int d0 = aux.d0;
        for (int i = et; i <= kWindow; i += 32 * kEpiWarps) {
          const int64_t di = (int64_t)d0 + i;
          aux.win[i] = di <= n_docs ? __ldg(coff + di) : INT64_MAX;
        }
        epi_bar();
        if (half == 0) {
          int dd = -1;
          if (c < C) {
            if (c < aux.win[kWindow]) {
              int lo = 0, hi = kWindow;  // win[lo] <= c < win[hi]
              while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (aux.win[mid] <= c) lo = mid; else hi = mid;
              }
              dd = d0 + lo;
            } else {  // more than kWindow documents in one tile (empty documents)
              int lo = d0, hi = n_docs;
              while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (__ldg(coff + mid) <= c) lo = mid; else hi = mid;
              }
              dd = lo;
            }
          }
          aux.doc_row[row] = dd;
        }
#pragma unroll
        for (int j = 0; j < K::HALF_N; ++j) acc[j] = 0.f;

        for (int h = 0; h < H; ++h, ++u) {
          const int st = u % K::STAGES;
          const uint32_t ph = (u / K::STAGES) & 1u;
          const int ab = u & 1;
          const uint32_t aph = (u >> 1) & 1u;
          // After a timeout the epilogue keeps walking its loop (skipping the
          // waits) so that every epilogue warp reaches every named barrier.
          if (!*abort_flag && !tc::mbar_wait(&aux.full[st], ph)) {
            record_error(status, MSA_ERR_TIMEOUT);
            *abort_flag = 1;
          }
          // |K̄_r[c, h]|^2 from this head's shared tile (swizzle only permutes
          // 16-byte pieces inside a row, which a sum of squares ignores)
          const unsigned char* arow = ring + st * K::STAGE + row * 128;
          float ss = 0.f;
          if (D == 128) {
            const unsigned char* base = arow + half * (kTile * 128);
#pragma unroll
            for (int j = 0; j < 8; ++j)
              ss += sumsq8(*reinterpret_cast<const uint4*>(base + j * 16));
          } else {
#pragma unroll
            for (int j = 0; j < 4; ++j)
              ss += sumsq8(*reinterpret_cast<const uint4*>(arow + (half * 4 + j) * 16));
          }
          aux.npart[u & 1][half][row] = ss;
          epi_bar();
          const float tot = aux.npart[u & 1][0][row] + aux.npart[u & 1][1][row];
          const float inv = 1.0f / fmaxf(sqrtf(tot), 1e-12f);
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(&aux.empty[st]);
          if (!*abort_flag && !tc::mbar_wait(&aux.accf[ab], aph)) {
            record_error(status, MSA_ERR_TIMEOUT);
            *abort_flag = 1;
          }
          tc::tc_fence_after();
          const uint32_t tbase = tmem + lane_addr + ab * N + half * K::HALF_N;
#pragma unroll
          for (int j = 0; j < K::HALF_N / 32; ++j) {
            uint32_t r[32];
            tc::tmem_ld32(tbase + j * 32, r);
            tc::tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) acc[j * 32 + i] = fmaf(inv, __uint_as_float(r[i]), acc[j * 32 + i]);
          }
          if (h + 1 < H) {
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&aux.acce[ab]);
          } else {
            // last head: park the head-mean cosines in the TMEM buffer just
            // read, then reduce them over tokens and documents
#pragma unroll
            for (int j = 0; j < K::HALF_N / 32; ++j) {
              float v[32];
#pragma unroll
              for (int i = 0; i < 32; ++i) v[i] = acc[j * 32 + i];
              tmem_st32(tbase + j * 32, v);
            }
            tmem_st_wait();
            const int dd = aux.doc_row[row];
            const bool valid = dd >= 0;
            // segment structure of the warp's rows (rows ascend with lanes)
            unsigned same = 0;
#pragma unroll
            for (int k = 0; k < 5; ++k) {
              const int off = 1 << k;
              const int od = __shfl_down_sync(0xffffffffu, dd, off);
              if (lane + off < 32 && od == dd) same |= 1u << k;
            }
            const int up = __shfl_up_sync(0xffffffffu, dd, 1);
            const bool head = valid && (lane == 0 || up != dd);
            int b = col_begin / T;
            int t = col_begin - b * T;
            float m = -INFINITY;
            for (int j = 0; j < K::HALF_N / 32; ++j) {
              uint32_t r[32];
              tc::tmem_ld32(tbase + j * 32, r);
              tc::tmem_ld_wait();
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const int col = col_begin + j * 32 + i;
                if (col >= NT) break;  // warp-uniform
                m = fmaxf(m, __uint_as_float(r[i]));
                const bool last_col = (j * 32 + i == K::HALF_N - 1) || (col + 1 >= NT) || (t + 1 == T);
                if (last_col) {
                  const uint32_t o = valid ? f2o(m) : 0u;
                  if (chunk_u && valid) atomicMax(chunk_u + (int64_t)b * C + c, o);
                  uint32_t x = o;
#pragma unroll
                  for (int k = 0; k < 5; ++k) {
                    const uint32_t y = __shfl_down_sync(0xffffffffu, x, 1 << k);
                    if (same & (1u << k)) x = max(x, y);
                  }
                  if (head) atomicMax(doc_u + (int64_t)b * n_docs + dd, x);
                  m = -INFINITY;
                }
                if (++t == T) { t = 0; ++b; }
              }
            }
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&aux.acce[ab]);
          }
        }
        epi_bar();  // doc_row / win are rewritten by the next tile
      }
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, K::TMEM_COLS);
  }
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

template <int N, int D>
int launch(int B, int T, int H, const __nv_bfloat16* qhat, int n_pad, const __nv_bfloat16* kr,
           int64_t C, const int64_t* coff, int n_docs, uint32_t* doc_u, uint32_t* chunk_u,
           int* status, cudaStream_t s) {
  using K = Cfg<N, D>;
  CUtensorMap tm_k, tm_q;
  if (!make_map(&tm_k, kr, D, H, C, (uint64_t)D * 2, (uint64_t)H * D * 2, 1, kTile))
    return note_cuda(cudaErrorInvalidValue);
  if (!make_map(&tm_q, qhat, D, n_pad, H, (uint64_t)D * 2, (uint64_t)n_pad * D * 2, N, 1))
    return note_cuda(cudaErrorInvalidValue);
  auto kern = route_tc_kernel<N, D>;
  int rc = note_cuda(
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)K::SMEM));
  if (rc) return rc;
  const int64_t n_tiles = (C + kTile - 1) / kTile;
  const int grid = (int)std::min<int64_t>(n_tiles, num_sms());
  const int NT = B * T;
  const int n_pass = n_pad / N;
  kern<<<grid, kThreads, K::SMEM, s>>>(tm_k, tm_q, H, NT, T, n_pass, C, n_tiles, coff, n_docs,
                                       doc_u, chunk_u, status);
  return check_launch();
}

}  // namespace

int64_t route_tc_columns(int64_t nt) {
  if (nt <= 64) return 64;
  if (nt <= 128) return 128;
  return (nt + 255) / 256 * 256;
}

int route_tc_launch(int B, int T, int H, int D, const __nv_bfloat16* qhat, int n_pad,
                    const __nv_bfloat16* kr, int64_t C, const int64_t* coff, int n_docs,
                    uint32_t* doc_u, uint32_t* chunk_u, int* status, cudaStream_t s) {
  const int N = n_pad <= 128 ? n_pad : 256;
  if (!aligned16(qhat) || !aligned16(kr)) return MSA_ERR_INVALID_ARG;
#define MSA_ROUTE_CASE(NN)                                                                      \
  if (N == NN)                                                                                  \
    return D == 64 ? launch<NN, 64>(B, T, H, qhat, n_pad, kr, C, coff, n_docs, doc_u, chunk_u,  \
                                    status, s)                                                  \
                   : launch<NN, 128>(B, T, H, qhat, n_pad, kr, C, coff, n_docs, doc_u, chunk_u, \
                                     status, s);
  MSA_ROUTE_CASE(64)
  MSA_ROUTE_CASE(128)
  MSA_ROUTE_CASE(256)
#undef MSA_ROUTE_CASE
  return MSA_ERR_UNSUPPORTED;
}

}  // namespace msa
