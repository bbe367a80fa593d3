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


// Ancestor masks of nodes [0, n): one lane per node walks its parent chain
// (parent < child) and writes the row's W words, highest word first.
__device__ __forceinline__ void write_masks(uint32_t* o_mask, int W, int n, const int32_t* n_parent, int lane) {
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
      j = n_parent[j];
    }
    row[cw] = bits;
    for (int w = cw - 1; w >= 0; --w) row[w] = 0u;
  }
}

// Pad rows [n, N): token / parent / depth / pos -1, score -inf, mask 0.
__device__ __forceinline__ void write_pads(int32_t* o_tok, int32_t* o_par, int32_t* o_dep, int32_t* o_pos,
                                           float* o_sc, uint32_t* o_mask, int W, int n, int N, int lane) {
  for (int i = n + lane; i < N; i += 32) {
    o_tok[i] = -1;
    o_par[i] = -1;
    o_dep[i] = -1;
    o_pos[i] = -1;
    o_sc[i] = -INFINITY;
    uint32_t* row = o_mask + (size_t)i * W;
    for (int w = 0; w < W; ++w) row[w] = 0u;
  }
}

// Loads one request's drafter output into shared memory and checks its
// precondition (finite, <= 0, non-increasing along k). Returns true if bad.
__device__ __forceinline__ bool load_drafter(const BuildParams& p, int b, float* lp, int32_t* tk, int lane) {
  const int DK = p.D * p.K;
  const float* lp_g = p.logp + (size_t)b * DK;
  const int32_t* tk_g = p.tok + (size_t)b * DK;
  bool bad = false;
  for (int e = lane; e < DK; e += 32) {
    const float v = lp_g[e];
    lp[e] = v;
    tk[e] = tk_g[e];
    if (!(v <= 0.0f) || isinf(v)) bad = true;  // NaN, +inf, > 0, -inf
    if ((e % p.K) != 0 && !(v <= lp_g[e - 1])) bad = true;
  }
  bad = __any_sync(DDT_FULL_MASK, bad);
  __syncwarp();
  return bad;
}

// Warp-wide winner among the lanes' local bests: score first (redux.sync on an
// order-preserving key), then depth, then the packed rank key. Returns the
// winning lane; `valid` marks lanes that hold a candidate.
__device__ __forceinline__ int warp_winner(bool valid, float bs, int bd, uint64_t bk, int lane) {
  const uint32_t so = valid ? float_order_key(bs) : 0u;
  const uint32_t top = __reduce_max_sync(DDT_FULL_MASK, so);
  uint32_t cand = __ballot_sync(DDT_FULL_MASK, valid && so == top);
  if (__popc(cand) > 1) {
    bool in = (cand >> lane) & 1u;
    const uint32_t dmin = __reduce_min_sync(DDT_FULL_MASK, in ? (uint32_t)bd : 0xffffffffu);
    cand = __ballot_sync(DDT_FULL_MASK, in && (uint32_t)bd == dmin);
    if (__popc(cand) > 1) {
      in = (cand >> lane) & 1u;
      const uint32_t khi = __reduce_min_sync(DDT_FULL_MASK, in ? (uint32_t)(bk >> 32) : 0xffffffffu);
      cand = __ballot_sync(DDT_FULL_MASK, in && (uint32_t)(bk >> 32) == khi);
      in = (cand >> lane) & 1u;
      const uint32_t klo = __reduce_min_sync(DDT_FULL_MASK, in ? (uint32_t)bk : 0xffffffffu);
      cand = __ballot_sync(DDT_FULL_MASK, in && (uint32_t)bk == klo);
    }
  }
  return __ffs(cand) - 1;
}

__global__ void __launch_bounds__(32) build_tree_kernel(BuildParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  pdl_wait();
  pdl_launch_dependents();
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
  const bool bad = load_drafter(p, b, s.lp, s.tk, lane);

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
      const int wl = warp_winner(bslot >= 0, bs, bd, bk, lane);
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
    write_masks(o_mask, W, n, s.n_parent, lane);
  }
  write_pads(o_tok, o_par, o_dep, o_pos, o_sc, o_mask, W, n, N, lane);
  if (lane == 0) {
    p.n_nodes[b] = n;
    if (p.dev_status) p.dev_status[b] = bad ? DDT_ERR_INPUT : DDT_OK;
  }
}


// Same search with the frontier in registers: slot f lives in lane f % 32,
// register f / 32 (SPL = slots per lane, N <= 32 * SPL). A pop then needs no
// shared-memory traffic: each lane scans its own registers, the winner's entry
// is broadcast with shuffles, and only the owner lanes of the (at most two)
// updated slots write.
template <int SPL>
__global__ void __launch_bounds__(32) build_tree_reg_kernel(BuildParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  pdl_wait();
  pdl_launch_dependents();
  const int b = blockIdx.x;
  const int lane = threadIdx.x;
  const int N = p.N, D = p.D, K = p.K, W = p.W;
  int32_t* n_parent = reinterpret_cast<int32_t*>(smem_raw);
  float* lp = reinterpret_cast<float*>(smem_raw + (size_t)N * 4);
  int32_t* tk = reinterpret_cast<int32_t*>(smem_raw + (size_t)N * 4 + (size_t)D * K * 4);
  const bool bad = load_drafter(p, b, lp, tk, lane);

  const int L = p.cache_len[b];
  int32_t* o_tok = p.node_tok + (size_t)b * N;
  int32_t* o_par = p.parent + (size_t)b * N;
  int32_t* o_dep = p.depth + (size_t)b * N;
  int32_t* o_pos = p.pos + (size_t)b * N;
  float* o_sc = p.score + (size_t)b * N;
  uint32_t* o_mask = p.mask + (size_t)b * N * W;

  int n = 0;
  if (!bad) {
    float f_sc[SPL], f_ps[SPL];
    int f_d[SPL], f_r[SPL], f_p[SPL];
    uint64_t f_k[SPL];
#pragma unroll
    for (int q = 0; q < SPL; ++q) {
      f_sc[q] = 0.0f; f_ps[q] = 0.0f; f_d[q] = 0; f_r[q] = 0; f_p[q] = 0; f_k[q] = 0ull;
    }
    if (lane == 0) {
      o_tok[0] = p.root_tok[b];
      o_par[0] = -1;
      o_dep[0] = 0;
      o_pos[0] = L;
      o_sc[0] = 0.0f;
      n_parent[0] = -1;
      f_sc[0] = __fadd_rn(0.0f, lp[0]);  // rank 0 at depth 1
      f_d[0] = 1;
    }
    int fsize = (N > 1) ? 1 : 0;
    n = 1;
    while (n < N && fsize > 0) {
      // lane-local best over this lane's slots
      int bj = -1;
      float bs = 0.0f;
      int bd = 0;
      uint64_t bk = 0ull;
#pragma unroll
      for (int q = 0; q < SPL; ++q) {
        if (32 * q + lane < fsize && (bj < 0 || better(f_sc[q], f_d[q], f_k[q], bs, bd, bk))) {
          bj = q; bs = f_sc[q]; bd = f_d[q]; bk = f_k[q];
        }
      }
      const int wl = warp_winner(bj >= 0, bs, bd, bk, lane);
      // the winner's remaining fields
      float ps_l = 0.0f;
      int r_l = 0, p_l = 0;
#pragma unroll
      for (int q = 0; q < SPL; ++q)
        if (q == bj) { ps_l = f_ps[q]; r_l = f_r[q]; p_l = f_p[q]; }
      const int wj = __shfl_sync(DDT_FULL_MASK, bj, wl);
      const float sc = __shfl_sync(DDT_FULL_MASK, bs, wl);
      const int dd = __shfl_sync(DDT_FULL_MASK, bd, wl);
      const uint64_t kk = __shfl_sync(DDT_FULL_MASK, bk, wl);
      const float psc = __shfl_sync(DDT_FULL_MASK, ps_l, wl);
      const int rr = __shfl_sync(DDT_FULL_MASK, r_l, wl);
      const int pp = __shfl_sync(DDT_FULL_MASK, p_l, wl);
      const int slot = 32 * wj + wl;
      const int i = n;
      if (lane == wl) {
        o_tok[i] = tk[(dd - 1) * K + rr];
        o_par[i] = pp;
        o_dep[i] = dd;
        o_pos[i] = L + dd;
        o_sc[i] = sc;
        n_parent[i] = pp;
      }
      const bool has_child = dd < D;
      const bool has_sib = rr + 1 < K;
      if (has_child && lane == wl) {  // first child takes the popped slot
        const float cs = __fadd_rn(sc, lp[dd * K]);
#pragma unroll
        for (int q = 0; q < SPL; ++q)
          if (q == wj) { f_sc[q] = cs; f_ps[q] = sc; f_d[q] = dd + 1; f_r[q] = 0; f_p[q] = i; f_k[q] = kk << p.bpl; }
      }
      if (has_sib) {  // next sibling: the popped slot, or a new one at the end
        const int t = has_child ? fsize : slot;
        if (lane == (t & 31)) {
          const float ss = __fadd_rn(psc, lp[(dd - 1) * K + rr + 1]);
          const int tj = t >> 5;
#pragma unroll
          for (int q = 0; q < SPL; ++q)
            if (q == tj) { f_sc[q] = ss; f_ps[q] = psc; f_d[q] = dd; f_r[q] = rr + 1; f_p[q] = pp; f_k[q] = kk + 1ull; }
        }
        if (has_child) ++fsize;
      }
      if (!has_child && !has_sib) {  // remove the popped slot: move the last entry into it
        const int last = fsize - 1;
        if (last != slot) {
          const int ll = last & 31, lj = last >> 5;
          float m_sc = 0.0f, m_ps = 0.0f;
          int m_d = 0, m_r = 0, m_p = 0;
          uint64_t m_k = 0ull;
#pragma unroll
          for (int q = 0; q < SPL; ++q)
            if (q == lj) { m_sc = f_sc[q]; m_ps = f_ps[q]; m_d = f_d[q]; m_r = f_r[q]; m_p = f_p[q]; m_k = f_k[q]; }
          m_sc = __shfl_sync(DDT_FULL_MASK, m_sc, ll);
          m_ps = __shfl_sync(DDT_FULL_MASK, m_ps, ll);
          m_d = __shfl_sync(DDT_FULL_MASK, m_d, ll);
          m_r = __shfl_sync(DDT_FULL_MASK, m_r, ll);
          m_p = __shfl_sync(DDT_FULL_MASK, m_p, ll);
          m_k = __shfl_sync(DDT_FULL_MASK, m_k, ll);
          if (lane == wl) {
#pragma unroll
            for (int q = 0; q < SPL; ++q)
              if (q == wj) { f_sc[q] = m_sc; f_ps[q] = m_ps; f_d[q] = m_d; f_r[q] = m_r; f_p[q] = m_p; f_k[q] = m_k; }
          }
        }
        --fsize;
      }
      ++n;
    }
    __syncwarp();
    write_masks(o_mask, W, n, n_parent, lane);
  }
  write_pads(o_tok, o_par, o_dep, o_pos, o_sc, o_mask, W, n, N, lane);
  if (lane == 0) {
    p.n_nodes[b] = n;
    if (p.dev_status) p.dev_status[b] = bad ? DDT_ERR_INPUT : DDT_OK;
  }
}

template <int SPL>
static int launch_reg(const BuildParams& p, cudaStream_t stream) {
  const size_t smem = (size_t)p.N * 4 + (size_t)p.D * p.K * 8;
  if (smem > 48 * 1024) {
    if (cudaFuncSetAttribute(build_tree_reg_kernel<SPL>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
      return DDT_ERR_CUDA;
  }
  return launch_pdl(build_tree_reg_kernel<SPL>, (unsigned)p.B, 32, smem, stream, p);
}

int launch_build_tree(const BuildParams& p, cudaStream_t stream) {
  if (p.N <= 32) return launch_reg<1>(p, stream);
  if (p.N <= 64) return launch_reg<2>(p, stream);
  if (p.N <= 128) return launch_reg<4>(p, stream);
  if (p.N <= 256) return launch_reg<8>(p, stream);
  const size_t smem = build_smem_bytes(p.N, p.D, p.K);
  if (smem > 48 * 1024) {
    if (cudaFuncSetAttribute(build_tree_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return DDT_ERR_CUDA;
  }
  return launch_pdl(build_tree_kernel, (unsigned)p.B, 32, smem, stream, p);
}

}  // namespace ddt
