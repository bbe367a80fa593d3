// C ABI entry points of libddt.so: host-side argument checks and dispatch to
// the CUDA kernels. Every check here is synchronous and launches nothing on
// failure; see include/ddt.h for the contract of each call.
#include <atomic>
#include <cstdint>

#include "ddt_kernels.cuh"

namespace ddt {

static int bits_per_level(int K) {
  int b = 0;
  while ((1 << b) < K) ++b;
  return b;
}

static bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

static std::atomic<uint64_t> g_wait_limit_ns{2000000000ull};

uint64_t wait_limit_ns() { return g_wait_limit_ns.load(std::memory_order_relaxed); }

}  // namespace ddt

extern "C" {

const char* ddt_status_string(int status) {
  switch (status) {
    case DDT_OK: return "DDT_OK";
    case DDT_ERR_INVALID_ARG: return "DDT_ERR_INVALID_ARG";
    case DDT_ERR_UNSUPPORTED: return "DDT_ERR_UNSUPPORTED";
    case DDT_ERR_CAPACITY: return "DDT_ERR_CAPACITY";
    case DDT_ERR_INPUT: return "DDT_ERR_INPUT";
    case DDT_ERR_CUDA: return "DDT_ERR_CUDA";
    case DDT_ERR_TIMEOUT: return "DDT_ERR_TIMEOUT";
    case DDT_ERR_BOUNDS: return "DDT_ERR_BOUNDS";
    default: return "DDT_UNKNOWN_STATUS";
  }
}

int ddt_version(void) { return 200; }

uint64_t ddt_set_wait_limit_ns(uint64_t ns) {
  const uint64_t v = ns == 0 ? 2000000000ull : (ns < 1000000ull ? 1000000ull : ns);
  return ddt::g_wait_limit_ns.exchange(v);
}

int ddt_drafter_topk(const void* logits, int logits_dtype, int V, int R, int K, float* logp, int32_t* tok,
                     int32_t* dev_status, cudaStream_t stream) {
  if (!logits || !logp || !tok) return DDT_ERR_INVALID_ARG;
  if (R < 1 || V < 1 || K < 1 || K > 32 || K > V) return DDT_ERR_INVALID_ARG;
  if (logits_dtype != DDT_F32 && logits_dtype != DDT_BF16) return DDT_ERR_INVALID_ARG;
  // up to 8 CTAs per row in a one-dimensional grid; slice bounds stay in int
  if (R > (1 << 28) - 1 || V > (1 << 30)) return DDT_ERR_UNSUPPORTED;
  ddt::DrafterParams p{};
  p.logits = logits;
  p.logits_dtype = logits_dtype;
  p.V = V;
  p.R = R;
  p.K = K;
  p.logp = logp;
  p.tok = tok;
  p.dev_status = dev_status;
  return ddt::launch_drafter_topk(p, stream);
}

int ddt_build_tree(const float* logp, const int32_t* tok, const int32_t* root_tok,
                   const int32_t* cache_len, int B, int D, int K, int N, int32_t* node_tok,
                   int32_t* parent, int32_t* depth, int32_t* pos, float* score, uint32_t* mask,
                   int32_t* n_nodes, int32_t* dev_status, cudaStream_t stream) {
  if (!logp || !tok || !root_tok || !cache_len || !node_tok || !parent || !depth || !pos ||
      !score || !mask || !n_nodes)
    return DDT_ERR_INVALID_ARG;
  if (B < 1 || D < 1 || D > 64 || K < 1 || K > 32 || N < 1 || N > 1024) return DDT_ERR_INVALID_ARG;
  const int bpl = ddt::bits_per_level(K);
  const int levels = D < N - 1 ? D : N - 1;
  if ((long long)bpl * levels > 64) return DDT_ERR_UNSUPPORTED;
  ddt::BuildParams p{logp, tok, root_tok, cache_len, B, D, K, N, (N + 31) / 32, bpl,
                     node_tok, parent, depth, pos, score, mask, n_nodes, dev_status};
  return ddt::launch_build_tree(p, stream);
}

size_t ddt_verify_attn_workspace_size(int B, int N, int H, int d_latent, int d_rope, int max_cache_len,
                                      int in_dtype) {
  if (B < 1 || N < 1 || H < 1 || max_cache_len < 0) return 0;
  if (ddt::tc_attn_supported(d_latent, d_rope, in_dtype))
    return ddt::tc_attn_workspace_bytes(B, N, H, max_cache_len);
  return 0;
}

int ddt_verify_attn(const void* q, const void* kv, int64_t kv_rows, const int64_t* cache_off,
                    const int32_t* cache_len, const uint32_t* mask, const int32_t* n_nodes, int B,
                    int N, int H, int d_latent, int d_rope, float scale, int max_cache_len,
                    int in_dtype, int out_dtype, void* out, float* lse, int32_t* dev_status, void* workspace,
                    size_t workspace_bytes, cudaStream_t stream) {
  if (!q || !kv || !cache_off || !cache_len || !mask || !n_nodes || !out) return DDT_ERR_INVALID_ARG;
  if (B < 1 || N < 1 || N > 1024 || H < 1 || d_latent < 1 || d_rope < 0 || max_cache_len < 0 ||
      kv_rows < 1)
    return DDT_ERR_INVALID_ARG;
  if (!(scale > 0.0f) || scale != scale) return DDT_ERR_INVALID_ARG;
  if ((in_dtype != DDT_F32 && in_dtype != DDT_BF16) || (out_dtype != DDT_F32 && out_dtype != DDT_BF16))
    return DDT_ERR_INVALID_ARG;
  const int d_qk = d_latent + d_rope;
  if (d_qk > 1024) return DDT_ERR_UNSUPPORTED;
  ddt::AttnParams p{q, kv, cache_off, cache_len, mask, n_nodes, B, N, H, d_latent, d_rope,
                    (N + 31) / 32, scale, in_dtype, out_dtype, out, lse, dev_status, kv_rows};
  if (ddt::tc_attn_supported(d_latent, d_rope, in_dtype)) {
    const size_t need = ddt::tc_attn_workspace_bytes(B, N, H, max_cache_len);
    if (workspace_bytes < need || (need > 0 && (!workspace || !ddt::aligned(workspace, 256))))
      return DDT_ERR_INVALID_ARG;
    if (!ddt::aligned(q, 16) || !ddt::aligned(kv, 16) || !ddt::aligned(out, 16)) return DDT_ERR_INVALID_ARG;
    return ddt::launch_attn_tc(p, max_cache_len, workspace, workspace_bytes, stream);
  }
  return ddt::launch_attn_simt(p, stream);
}

size_t ddt_accept_compact_workspace_size(int B, int N, int V) {
  if (B < 1 || N < 1 || V < 1) return 0;
  return ddt::accept_workspace_bytes(B, N, V);
}

int ddt_accept_compact(const void* logits, int logits_dtype, int V, const int32_t* node_tok,
                       const int32_t* parent, const int32_t* n_nodes, int B, int N, void* kv,
                       int64_t kv_rows, int kv_dtype, int row_elems, int n_layers, int64_t layer_stride_rows,
                       const int64_t* cache_off, int32_t* cache_len, const int32_t* cache_cap,
                       int32_t* am, int32_t* acc_len, int32_t* acc_nodes, int32_t* out_tok,
                       int32_t* bonus, int32_t* dev_status, void* workspace, size_t workspace_bytes,
                       cudaStream_t stream) {
  if (!logits || !node_tok || !parent || !n_nodes || !kv || !cache_off || !cache_len || !cache_cap ||
      !acc_len || !acc_nodes || !out_tok || !bonus || !workspace)
    return DDT_ERR_INVALID_ARG;
  if (B < 1 || N < 1 || N > 1024 || V < 1 || row_elems < 1 || n_layers < 1 || layer_stride_rows < 0)
    return DDT_ERR_INVALID_ARG;
  if (n_layers > 1 && layer_stride_rows < 1) return DDT_ERR_INVALID_ARG;
  if (kv_rows < 1) return DDT_ERR_INVALID_ARG;
  if ((logits_dtype != DDT_F32 && logits_dtype != DDT_BF16) || (kv_dtype != DDT_F32 && kv_dtype != DDT_BF16))
    return DDT_ERR_INVALID_ARG;
  const int elt = kv_dtype == DDT_F32 ? 4 : 2;
  const long long row_bytes = (long long)row_elems * elt;
  if (row_bytes % 4 != 0 || row_bytes > (1 << 20)) return DDT_ERR_INVALID_ARG;
  if (!ddt::aligned(kv, 4) || !ddt::aligned(workspace, 256)) return DDT_ERR_INVALID_ARG;
  if (workspace_bytes < ddt::accept_workspace_bytes(B, N, V)) return DDT_ERR_INVALID_ARG;
  ddt::AcceptParams p{};
  p.logits = logits;
  p.logits_dtype = logits_dtype;
  p.V = V;
  p.node_tok = node_tok;
  p.parent = parent;
  p.n_nodes = n_nodes;
  p.B = B;
  p.N = N;
  p.kv = static_cast<unsigned char*>(kv);
  p.kv_rows = kv_rows;
  p.row_bytes = (int)row_bytes;
  p.n_layers = n_layers;
  p.layer_stride_bytes = layer_stride_rows * row_bytes;
  p.cache_off = cache_off;
  p.cache_len = cache_len;
  p.cache_cap = cache_cap;
  p.am = am;
  p.acc_len = acc_len;
  p.acc_nodes = acc_nodes;
  p.out_tok = out_tok;
  p.bonus = bonus;
  p.dev_status = dev_status;
  return ddt::launch_accept_compact(p, workspace, stream);
}

int ddt_accept_compact_lmhead(const void* hidden, const void* w_vocab, int d_model, int V, const int32_t* node_tok,
                              const int32_t* parent, const int32_t* n_nodes, int B, int N, void* kv, int64_t kv_rows,
                              int kv_dtype, int row_elems, int n_layers, int64_t layer_stride_rows,
                              const int64_t* cache_off, int32_t* cache_len, const int32_t* cache_cap, int32_t* am,
                              int32_t* acc_len, int32_t* acc_nodes, int32_t* out_tok, int32_t* bonus,
                              int32_t* dev_status, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (!hidden || !w_vocab || !node_tok || !parent || !n_nodes || !kv || !cache_off || !cache_len || !cache_cap ||
      !acc_len || !acc_nodes || !out_tok || !bonus || !workspace)
    return DDT_ERR_INVALID_ARG;
  if (B < 1 || N < 1 || N > 1024 || V < 1 || d_model < 1 || row_elems < 1 || n_layers < 1 || layer_stride_rows < 0)
    return DDT_ERR_INVALID_ARG;
  if (n_layers > 1 && layer_stride_rows < 1) return DDT_ERR_INVALID_ARG;
  if (kv_rows < 1) return DDT_ERR_INVALID_ARG;
  if (kv_dtype != DDT_F32 && kv_dtype != DDT_BF16) return DDT_ERR_INVALID_ARG;
  const int elt = kv_dtype == DDT_F32 ? 4 : 2;
  const long long row_bytes = (long long)row_elems * elt;
  if (row_bytes % 4 != 0 || row_bytes > (1 << 20)) return DDT_ERR_INVALID_ARG;
  if (!ddt::aligned(kv, 4) || !ddt::aligned(workspace, 256)) return DDT_ERR_INVALID_ARG;
  if (workspace_bytes < ddt::accept_workspace_bytes(B, N, V)) return DDT_ERR_INVALID_ARG;
  if (!ddt::lmhead_supported(d_model, V, hidden, w_vocab)) return DDT_ERR_UNSUPPORTED;
  if ((long long)B * N > (1LL << 30) || (long long)V * d_model > (1LL << 40)) return DDT_ERR_UNSUPPORTED;
  ddt::AcceptParams p{};
  p.logits = nullptr;
  p.logits_dtype = DDT_BF16;
  p.V = V;
  p.node_tok = node_tok;
  p.parent = parent;
  p.n_nodes = n_nodes;
  p.B = B;
  p.N = N;
  p.kv = static_cast<unsigned char*>(kv);
  p.kv_rows = kv_rows;
  p.row_bytes = (int)row_bytes;
  p.n_layers = n_layers;
  p.layer_stride_bytes = layer_stride_rows * row_bytes;
  p.cache_off = cache_off;
  p.cache_len = cache_len;
  p.cache_cap = cache_cap;
  p.am = am;
  p.acc_len = acc_len;
  p.acc_nodes = acc_nodes;
  p.out_tok = out_tok;
  p.bonus = bonus;
  p.dev_status = dev_status;
  const int st = ddt::launch_lmhead_argmax(hidden, w_vocab, d_model, V, B, N, n_nodes, workspace, stream);
  if (st != DDT_OK) return st;
  return ddt::launch_accept_walk(p, workspace, stream);
}

int ddt_accept_compact_noalloc(const void* logits, int logits_dtype, int V, const int32_t* node_tok,
                               const int32_t* parent, const int32_t* n_nodes, int B, int N, void* kv,
                               int64_t kv_rows, int kv_dtype, int row_elems, int n_layers, int64_t layer_stride_rows, const int64_t* cache_off,
                               int32_t* cache_len, const int32_t* cache_cap, int32_t* am, int32_t* acc_len,
                               int32_t* acc_nodes, int32_t* out_tok, int32_t* bonus, int32_t* dev_status,
                               cudaStream_t stream) {
  if (!logits || !node_tok || !parent || !n_nodes || !kv || !cache_off || !cache_len || !cache_cap || !acc_len ||
      !acc_nodes || !out_tok || !bonus)
    return DDT_ERR_INVALID_ARG;
  if (B < 1 || N < 1 || N > 1024 || V < 1 || row_elems < 1 || n_layers < 1 || layer_stride_rows < 0)
    return DDT_ERR_INVALID_ARG;
  if (n_layers > 1 && layer_stride_rows < 1) return DDT_ERR_INVALID_ARG;
  if (kv_rows < 1) return DDT_ERR_INVALID_ARG;
  if ((logits_dtype != DDT_F32 && logits_dtype != DDT_BF16) || (kv_dtype != DDT_F32 && kv_dtype != DDT_BF16))
    return DDT_ERR_INVALID_ARG;
  const int elt = kv_dtype == DDT_F32 ? 4 : 2;
  const long long row_bytes = (long long)row_elems * elt;
  if (row_bytes % 4 != 0 || row_bytes > (1 << 20)) return DDT_ERR_INVALID_ARG;
  if (!ddt::aligned(kv, 4)) return DDT_ERR_INVALID_ARG;
  ddt::AcceptParams p{};
  p.logits = logits;
  p.logits_dtype = logits_dtype;
  p.V = V;
  p.node_tok = node_tok;
  p.parent = parent;
  p.n_nodes = n_nodes;
  p.B = B;
  p.N = N;
  p.kv = static_cast<unsigned char*>(kv);
  p.kv_rows = kv_rows;
  p.row_bytes = (int)row_bytes;
  p.n_layers = n_layers;
  p.layer_stride_bytes = layer_stride_rows * row_bytes;
  p.cache_off = cache_off;
  p.cache_len = cache_len;
  p.cache_cap = cache_cap;
  p.am = am;
  p.acc_len = acc_len;
  p.acc_nodes = acc_nodes;
  p.out_tok = out_tok;
  p.bonus = bonus;
  p.dev_status = dev_status;
  return ddt::launch_accept_compact_noalloc(p, stream);
}

}  // extern "C"
