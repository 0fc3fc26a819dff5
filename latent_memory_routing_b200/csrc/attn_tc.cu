// bf16 prefill attention on the tcgen05 tensor cores.
#include "attn_tc.cuh"
#include "msa_common.cuh"

namespace msa {

bool attn_tc_supported(int, int, int, int, int, int, int) { return false; }
size_t attn_tc_workspace_size(int, int, int, int, int, int, int) { return 0; }
int attn_tc_launch(int, int, int, int, int, int, const void*, const void*, const void*,
                   const int32_t*, int, const void*, const void*, int, float, float, void*, void*,
                   cudaStream_t) {
  return MSA_ERR_UNSUPPORTED;
}

}  // namespace msa
