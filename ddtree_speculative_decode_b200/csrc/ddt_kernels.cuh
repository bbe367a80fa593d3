// Internal interface between the C ABI layer (ddt_api.cu) and the kernels.
#pragma once

#include "ddt_common.cuh"

namespace ddt {

// ---- tree build -------------------------------------------------------------
struct BuildParams {
  const float* logp;
  const int32_t* tok;
  const int32_t* root_tok;
  const int32_t* cache_len;
  int B, D, K, N, W, bpl;
  int32_t* node_tok;
  int32_t* parent;
  int32_t* depth;
  int32_t* pos;
  float* score;
  uint32_t* mask;
  int32_t* n_nodes;
  int32_t* dev_status;
};
int launch_build_tree(const BuildParams& p, cudaStream_t stream);

// ---- accept + compaction ------------------------------------------------------
struct AcceptParams {
  const void* logits;
  int logits_dtype;
  int V;
  const int32_t* node_tok;
  const int32_t* parent;
  const int32_t* n_nodes;
  int B, N;
  unsigned char* kv;
  int64_t kv_rows;              // rows in the pool (all layers)
  int row_bytes;
  int n_layers;
  int64_t layer_stride_bytes;
  const int64_t* cache_off;
  int32_t* cache_len;
  const int32_t* cache_cap;
  int32_t* am;
  int32_t* acc_len;
  int32_t* acc_nodes;
  int32_t* out_tok;
  int32_t* bonus;
  int32_t* dev_status;
  unsigned long long* rowkey;   // [B*N] packed (value, ~index) row maxima (zero between calls)
  const int* status_word;       // nullable: non-zero when the argmax producer gave up a wait
  int* abort;                   // the same word, for the argmax kernel's bounded waits
  unsigned* work;               // argmax work counter: chunks of slices handed out (zero between calls)
  uint64_t wait_ns;
  int tma;                      // logits rows stream by bulk copies (16-byte aligned rows)
  int layers_apart;             // several layers: a second kernel moves the rows
};
size_t accept_workspace_bytes(int B, int N, int V);
int launch_accept_compact(AcceptParams p, void* workspace, cudaStream_t stream);
int launch_accept_walk(AcceptParams p, void* workspace, cudaStream_t stream);
size_t accept_noalloc_scratch_bytes();
int launch_accept_compact_noalloc(AcceptParams p, cudaStream_t stream);

// ---- target LM head folded into the accept argmax ------------------------------
bool lmhead_supported(int d_model, int V, const void* hidden, const void* w_vocab);
// row keys of the workspace (ddt_accept_compact layout) from hidden [B*N][d] x w [V][d]
int launch_lmhead_argmax(const void* hidden, const void* w_vocab, int d_model, int V, int B, int N,
                         const int32_t* n_nodes, void* workspace, cudaStream_t stream);

// ---- drafter proposals --------------------------------------------------------
struct DrafterParams {
  const void* logits;   // [R][V]
  int logits_dtype;
  int V, R, K;
  float* logp;          // [R][K]
  int32_t* tok;         // [R][K]
  int32_t* dev_status;  // [R], nullable
  int vec;              // rows are 16-byte aligned
  int C;                // CTAs (one cluster) per row
  int chunk;            // logits per CTA (a multiple of 8)
};
int launch_drafter_topk(DrafterParams p, cudaStream_t stream);

// ---- verify attention -------------------------------------------------------
struct AttnParams {
  const void* q;
  const void* kv;
  const int64_t* cache_off;
  const int32_t* cache_len;
  const uint32_t* mask;
  const int32_t* n_nodes;
  int B, N, H, d_l, d_r, W;
  float scale;
  int in_dtype, out_dtype;
  void* out;
  float* lse;
  int32_t* dev_status;  // [B], nullable: DDT_OK or DDT_ERR_BOUNDS
  int64_t kv_rows;
};
int launch_attn_simt(const AttnParams& p, cudaStream_t stream);

bool tc_attn_supported(int d_l, int d_r, int in_dtype);
size_t tc_attn_workspace_bytes(int B, int N, int H, int max_cache_len);
int launch_attn_tc(const AttnParams& p, int max_cache_len, void* workspace,
                   size_t workspace_bytes, cudaStream_t stream);

}  // namespace ddt
