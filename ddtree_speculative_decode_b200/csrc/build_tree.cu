// Best-first draft-tree build: one warp per request.
//
// What it computes is fixed in ddt.h (ddt_build_tree): the first N - 1 rank
// paths in (score desc, depth asc, ranks lexicographic asc) order, scores as
// left-to-right float32 sums of the drafter's per-depth log-probs
// ("ddtree_speculative_decode_test_capstone", section "What the Test
// Validated"; "autoregressive_test_driver_kdtree_engine", section "The Broader
// Context": a GPU best-first builder replacing a per-request heapq).
//
// Design. The frontier of a best-first search over sorted candidates never
// holds more than (pops + 1) entries, so it fits a shared-memory array of N
// slots. Each pop is a warp-wide argmax over the frontier: every lane scans
// its slots (slot % 32 == lane), then the warp settles the winner with
// redux.sync on an order-preserving 32-bit score key, falling back to depth
// and the packed rank-tuple key only when scores tie. The popped path pushes
// at most two successors (its first child and its next sibling), which reuse
// the popped slot and, if needed, one new slot. Lexicographic rank order is a
// packed integer: ceil(log2 K) bits per level, first level most significant,
// so equal-depth paths compare as integers. Ancestor masks are filled after
// selection, one lane per node, by walking parent pointers (parent < child).
#include "ddt_kernels.cuh"

namespace ddt {

// Shared-memory layout for one warp (one request), capacity N.
struct BuildSmem {
  float* f_score;     // frontier: path score
  float* f_pscore;    // frontier: score of the path's parent (for siblings)
  int32_t* f_depth;   // frontier: path depth
  int32_t* f_rank;    // frontier: last rank
  int32_t* f_parent;  // frontier: node index of the path's parent
  uint64_t* f_key;    // frontier: packed rank tuple
  int32_t* n_parent;  // selected nodes: parent
  float* lp;          // drafter log-probs [D][K]
  int32_t* tk;        // drafter tokens [D][K]
};

__host__ __device__ inline size_t build_smem_bytes(int N, int D, int K) {
  size_t b = 0;
  b += (size_t)N * 8;                  // f_key
  b += (size_t)N * 4 * 5;              // f_score f_pscore f_depth f_rank f_parent
  b += (size_t)N * 4;                  // n_parent
  b += (size_t)D * K * 8;              // lp + tk
  return b;
}

__device__ __forceinline__ bool better(float sa, int da, uint64_t ka, float sb, int db, uint64_t kb) {
  if (sa != sb) return sa > sb;
  if (da != db) return da < db;
  return ka < kb;
}

__global__ void __launch_bounds__(32) build_tree_kernel(BuildParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int b = blockIdx.x;
  const int lane = threadIdx.x;
  const int N = p.N, D = p.D, K = p.K, W = p.W;

  BuildSmem s;
  unsigned char* cur = smem_raw;
  s.f_key = reinterpret_cast<uint64_t*>(cur); cur += (size_t)N * 8;
  s.f_score = reinterpret_cast<float*>(cur); cur += (size_t)N * 4;
  s.f_pscore = reinterpret_cast<float*>(cur); cur += (size_t)N * 4;
  s.f_depth = reinterpret_cast<int32_t*>(cur); cur += (size_t)N * 4;
  s.f_rank = reinterpret_cast<int32_t*>(cur); cur += (size_t)N * 4;
  s.f_parent = reinterpret_cast<int32_t*>(cur); cur += (size_t)N * 4;
  s.n_parent = reinterpret_cast<int32_t*>(cur); cur += (size_t)N * 4;
  s.lp = reinterpret_cast<float*>(cur); cur += (size_t)D * K * 4;
  s.tk = reinterpret_cast<int32_t*>(cur);

  // ---- load drafter output, check its precondition -------------------------
  const float* lp_g = p.logp + (size_t)b * D * K;
  const int32_t* tk_g = p.tok + (size_t)b * D * K;
  bool bad = false;
  for (int e = lane; e < D * K; e += 32) {
    float v = lp_g[e];
    s.lp[e] = v;
    s.tk[e] = tk_g[e];
    if (!(v <= 0.0f) || isinf(v)) bad = true;  // NaN, +inf, > 0, -inf
    if ((e % K) != 0 && !(v <= lp_g[e - 1])) bad = true;
  }
  bad = __any_sync(DDT_FULL_MASK, bad);
  __syncwarp();

  const int L = p.cache_len[b];
  int32_t* o_tok = p.node_tok + (size_t)b * N;
  int32_t* o_par = p.parent + (size_t)b * N;
  int32_t* o_dep = p.depth + (size_t)b * N;
  int32_t* o_pos = p.pos + (size_t)b * N;
  float* o_sc = p.score + (size_t)b * N;
  uint32_t* o_mask = p.mask + (size_t)b * N * W;

  int n = 0;
  if (!bad) {
    // ---- root + best-first pops --------------------------------------------
    if (lane == 0) {
      o_tok[0] = p.root_tok[b];
      o_par[0] = -1;
      o_dep[0] = 0;
      o_pos[0] = L;
      o_sc[0] = 0.0f;
      s.n_parent[0] = -1;
      // first candidate: rank 0 at depth 1
      s.f_score[0] = __fadd_rn(0.0f, s.lp[0]);
      s.f_pscore[0] = 0.0f;
      s.f_depth[0] = 1;
      s.f_rank[0] = 0;
      s.f_parent[0] = 0;
      s.f_key[0] = 0ull;
    }
    __syncwarp();
    int fsize = (N > 1) ? 1 : 0;
    n = 1;
    while (n < N && fsize > 0) {
      // lane-local best
      float bs = 0.0f;
      int bd = 0;
      uint64_t bk = 0;
      int bslot = -1;
      for (int f = lane; f < fsize; f += 32) {
        float sc = s.f_score[f];
        int dd = s.f_depth[f];
        uint64_t kk = s.f_key[f];
        if (bslot < 0 || better(sc, dd, kk, bs, bd, bk)) {
          bs = sc; bd = dd; bk = kk; bslot = f;
        }
      }
      // warp-wide winner: score, then depth, then packed ranks
      uint32_t so = bslot >= 0 ? float_order_key(bs) : 0u;
      uint32_t top = __reduce_max_sync(DDT_FULL_MASK, so);
      uint32_t cand = __ballot_sync(DDT_FULL_MASK, bslot >= 0 && so == top);
      if (__popc(cand) > 1) {
        bool in = (cand >> lane) & 1u;
        uint32_t dmin = __reduce_min_sync(DDT_FULL_MASK, in ? (uint32_t)bd : 0xffffffffu);
        cand = __ballot_sync(DDT_FULL_MASK, in && (uint32_t)bd == dmin);
        if (__popc(cand) > 1) {
          in = (cand >> lane) & 1u;
          uint32_t khi = __reduce_min_sync(DDT_FULL_MASK, in ? (uint32_t)(bk >> 32) : 0xffffffffu);
          cand = __ballot_sync(DDT_FULL_MASK, in && (uint32_t)(bk >> 32) == khi);
          in = (cand >> lane) & 1u;
          uint32_t klo = __reduce_min_sync(DDT_FULL_MASK, in ? (uint32_t)bk : 0xffffffffu);
          cand = __ballot_sync(DDT_FULL_MASK, in && (uint32_t)bk == klo);
        }
      }
      const int wl = __ffs(cand) - 1;
      const int slot = __shfl_sync(DDT_FULL_MASK, bslot, wl);
      if (lane == 0) {
        const float sc = s.f_score[slot];
        const float psc = s.f_pscore[slot];
        const int dd = s.f_depth[slot];
        const int rr = s.f_rank[slot];
        const int pp = s.f_parent[slot];
        const uint64_t kk = s.f_key[slot];
        const int i = n;
        o_tok[i] = s.tk[(dd - 1) * K + rr];
        o_par[i] = pp;
        o_dep[i] = dd;
        o_pos[i] = L + dd;
        o_sc[i] = sc;
        s.n_parent[i] = pp;
        bool used = false;
        if (dd < D) {  // first child takes the popped slot
          s.f_score[slot] = __fadd_rn(sc, s.lp[dd * K]);
          s.f_pscore[slot] = sc;
          s.f_depth[slot] = dd + 1;
          s.f_rank[slot] = 0;
          s.f_parent[slot] = i;
          s.f_key[slot] = kk << p.bpl;
          used = true;
        }
        if (rr + 1 < K) {  // next sibling
          const int t = used ? fsize : slot;
          s.f_score[t] = __fadd_rn(psc, s.lp[(dd - 1) * K + rr + 1]);
          s.f_pscore[t] = psc;
          s.f_depth[t] = dd;
          s.f_rank[t] = rr + 1;
          s.f_parent[t] = pp;
          s.f_key[t] = kk + 1ull;
          if (used) ++fsize;
          used = true;
        }
        if (!used) {  // remove: move the last entry into the hole
          const int last = fsize - 1;
          if (last != slot) {
            s.f_score[slot] = s.f_score[last];
            s.f_pscore[slot] = s.f_pscore[last];
            s.f_depth[slot] = s.f_depth[last];
            s.f_rank[slot] = s.f_rank[last];
            s.f_parent[slot] = s.f_parent[last];
            s.f_key[slot] = s.f_key[last];
          }
          --fsize;
        }
      }
      fsize = __shfl_sync(DDT_FULL_MASK, fsize, 0);
      ++n;
      __syncwarp();
    }
    // ---- ancestor masks: one lane per node, walk parents -----------------
    for (int i = lane; i < n; i += 32) {
      uint32_t* row = o_mask + (size_t)i * W;
      for (int w = (i >> 5) + 1; w < W; ++w) row[w] = 0u;
      int cw = i >> 5;
      uint32_t bits = 0u;
      int j = i;
      while (j >= 0) {
        const int w = j >> 5;
        while (w < cw) {
          row[cw] = bits;
          bits = 0u;
          --cw;
        }
        bits |= 1u << (j & 31);
        j = s.n_parent[j];
      }
      row[cw] = bits;
      for (int w = cw - 1; w >= 0; --w) row[w] = 0u;
    }
  }
  // ---- pad rows -------------------------------------------------------------
  for (int i = n + lane; i < N; i += 32) {
    o_tok[i] = -1;
    o_par[i] = -1;
    o_dep[i] = -1;
    o_pos[i] = -1;
    o_sc[i] = -INFINITY;
    uint32_t* row = o_mask + (size_t)i * W;
    for (int w = 0; w < W; ++w) row[w] = 0u;
  }
  if (lane == 0) {
    p.n_nodes[b] = n;
    if (p.dev_status) p.dev_status[b] = bad ? DDT_ERR_INPUT : DDT_OK;
  }
}

int launch_build_tree(const BuildParams& p, cudaStream_t stream) {
  const size_t smem = build_smem_bytes(p.N, p.D, p.K);
  if (smem > 48 * 1024) {
    if (cudaFuncSetAttribute(build_tree_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return DDT_ERR_CUDA;
  }
  build_tree_kernel<<<p.B, 32, smem, stream>>>(p);
  return launch_status();
}

}  // namespace ddt
