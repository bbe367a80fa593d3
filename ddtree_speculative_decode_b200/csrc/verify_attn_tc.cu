// Tensor-core (tcgen05 / TMEM / TMA) tree-verify attention for bf16 inputs
// with the Kimi K2.6 MLA shape (512-d latent + 64-d RoPE).
#include "ddt_kernels.cuh"

namespace ddt {

bool tc_attn_supported(int d_l, int d_r, int in_dtype) {
  (void)d_l; (void)d_r; (void)in_dtype;
  return false;
}

size_t tc_attn_workspace_bytes(int B, int N, int H, int max_cache_len) {
  (void)B; (void)N; (void)H; (void)max_cache_len;
  return 0;
}

int launch_attn_tc(const AttnParams& p, int64_t kv_rows, int max_cache_len, void* workspace,
                   size_t workspace_bytes, cudaStream_t stream) {
  (void)p; (void)kv_rows; (void)max_cache_len; (void)workspace; (void)workspace_bytes; (void)stream;
  return DDT_ERR_UNSUPPORTED;
}

}  // namespace ddt
