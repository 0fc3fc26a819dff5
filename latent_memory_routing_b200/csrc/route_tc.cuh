// bf16 routing scan on the tcgen05 tensor cores (route_tc.cu).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace msa {

// Query columns of one pass over the bank and the padded column count of
// the normalised-query workspace: B*T <= 256 is padded to 64, 128 or 256
// columns (one pass); larger B*T to a multiple of 256 (one pass per 256).
int64_t route_tc_columns(int64_t n_queries_tokens);

// Scans the whole bank once per pass.  qhat: [H][n_pad][D] bf16, each row
// Q_r / max(|Q_r|, eps) / H (rows >= B*T zero).  kr: [C][H][D] bf16.
// doc_u / chunk_u: order-preserving uint32 maxima, pre-set to -inf.
// `prepared`: kr rows are already unit-normalised (msa_route_prepare_bank);
// otherwise the kernel normalises them in shared memory.
int route_tc_launch(int B, int T, int H, int D, const __nv_bfloat16* qhat, int n_pad,
                    const __nv_bfloat16* kr, int64_t C, const int64_t* chunk_off,
                    int n_docs, uint32_t* doc_u, uint32_t* chunk_u, int* status,
                    bool prepared, cudaStream_t s);

// The same scan (raw bank) keeping, per (query b, document d), the first
// maximiser of the chunk-token cosine instead of the maximum: doc_key
// [B][n_docs] (pre-set to 0) receives (f2o(score) << 32) |
// ~((c - chunk_off[d]) * T + t); needs (chunks of any document) * T < 2^32.
int route_tc_argmax_launch(int B, int T, int H, int D, const __nv_bfloat16* qhat, int n_pad,
                           const __nv_bfloat16* kr, int64_t C, const int64_t* chunk_off,
                           int n_docs, unsigned long long* doc_key, int* status, cudaStream_t s);

// Normalised, head-major query columns for the tensor-core scan: qhat
// [H][n_pad][D] bf16 = Q_r / max(|Q_r|, 1e-12) / H, rows >= NT zero.
int route_prep_bf16_launch(int NT, int H, int D, int n_pad, const __nv_bfloat16* q_r,
                           __nv_bfloat16* qhat, cudaStream_t s);

// dst[r] = src[r] / max(|src[r]|, 1e-12) for n_rows rows of D bf16.
int route_prepare_bank_launch(int64_t n_rows, int D, const __nv_bfloat16* src,
                              __nv_bfloat16* dst, cudaStream_t s);

}  // namespace msa
