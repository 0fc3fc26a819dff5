// bf16 prefill attention on the tcgen05 tensor cores (attn_tc.cu).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace msa {

// True when the tensor-core prefill kernel takes this shape.
bool attn_tc_supported(int B, int T, int T_loc, int Hq, int H, int D, int m_cap);
size_t attn_tc_workspace_size(int B, int T, int T_loc, int Hq, int H, int D, int m_cap);
int attn_tc_launch(int B, int T, int T_loc, int Hq, int H, int D, const void* q,
                   const void* k_mem, const void* v_mem, const int32_t* mem_len, int m_cap,
                   const void* k_loc, const void* v_loc, int pos0, float rope_base, float qscale,
                   void* out, void* ws, cudaStream_t s);

// bf16 decode (T = 1) on the CUDA cores, streaming K/V once (attn_decode.cu).
bool attn_decode_supported(int T, int Hq, int H, int D);
size_t attn_decode_workspace_size(int B, int T_loc, int Hq, int H, int D, int m_cap);
int attn_decode_launch(int B, int T_loc, int Hq, int H, int D, const void* q, const void* k_mem,
                       const void* v_mem, const int32_t* mem_len, int m_cap, const void* k_loc,
                       const void* v_loc, int pos0, float rope_base, float qscale, void* out,
                       void* ws, cudaStream_t s);

// Tensor map of a bf16 [rows][heads][D] array viewed as dims {D, heads,
// rows}, 128-byte swizzle, box {64, bh, br}: 64-element K blocks of br rows,
// the layout of a K-major (or, read the other way, MN-major) UMMA operand.
bool tma_map_sw128_bf16(CUtensorMap* m, const void* ptr, int D, int heads, int64_t rows, int bh,
                        int br);

// Memory read straight from the pooled bank (fused assemble + attend): per
// query b, groups[b * max_groups + i] = (first bank row, rows of the group
// that belong to its document, 1..8) for i < n_groups[b], in rank order.
struct FusedMemory {
  const int2* groups;
  const int32_t* n_groups;
  int max_groups;
  const void* k_bar;
  const void* v_bar;
  int64_t n_chunks;
};

// bf16 decode on the tcgen05 tensor cores (attn_decode_tc.cu).
bool attn_decode_tc_supported(int T, int Hq, int H, int D);
size_t attn_decode_tc_workspace_size(int B, int T_loc, int Hq, int H, int D, int m_cap);
int attn_decode_tc_launch(int B, int T_loc, int Hq, int H, int D, const void* q,
                          const void* k_mem, const void* v_mem, const int32_t* mem_len,
                          int m_cap, const void* k_loc, const void* v_loc, int pos0,
                          float rope_base, float qscale, void* out, void* ws, cudaStream_t s);
size_t attn_decode_tc_fused_workspace_size(int B, int T_loc, int Hq, int H, int max_groups);
size_t attn_tc_fused_workspace_size(int B, int T, int T_loc, int Hq, int H, int D,
                                    int max_groups);
int attn_tc_launch_fused(int B, int T, int T_loc, int Hq, int H, int D, const void* q,
                         const FusedMemory& fm, const void* k_loc, const void* v_loc, int pos0,
                         float rope_base, float qscale, void* out, void* ws, cudaStream_t s);
int attn_decode_tc_launch_fused(int B, int T_loc, int Hq, int H, int D, const void* q,
                                const FusedMemory& fm, const void* k_loc, const void* v_loc,
                                int pos0, float rope_base, float qscale, void* out, void* ws,
                                cudaStream_t s);

// Tensor map of a bf16 [rows][heads][D] array viewed as dims {D, heads,
// rows}, no swizzle, box {D, 1, br}: one head's D-vector of br consecutive
// rows, stored densely (D * 2 bytes per row).  False if the driver's encoder
// is unavailable or rejects the shape.
bool tma_map_rows_bf16(CUtensorMap* m, const void* ptr, int D, int heads, int64_t rows, int br);

// Merges n_split partial results (unnormalised O in fp32, (max, sum) in the
// base-2 exponent domain) of each (query, head, token) row into bf16 out.
int attn_combine_bf16(int B, int T, int Hq, int D, int n_split, const float* part_o,
                      const float2* part_ml, void* out, cudaStream_t s);

}  // namespace msa
