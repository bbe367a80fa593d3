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


// ---------------------------------------------------------------------------
// Sorted-frontier variant (the default for N <= 256).
//
// The frontier is kept sorted across the warp: entry f lives in lane f % 32,
// register f / 32, and entry 0 is the best. A pop is "take entry 0"; its (at
// most two) successors are merged into the remaining entries in one step:
// two ballots count how many remaining entries beat each successor, which
// fixes every lane's source (old f+1, old f, old f-1 or a successor), and one
// shuffle per word moves the entries. Entries that can no longer be popped
// (beyond the number of pops left) are dropped, which keeps the frontier
// within min(pops + 1, N - 1 - pops) <= 32 * SPL entries for N <= 64 * SPL.
//
// An entry is five 32-bit words: hi = order key of the score (scores are
// <= 0, so the key is the complement of the bits of score + 0, which maps -0
// to +0; larger is better), aux = (127 - depth) << 24 | last rank << 16 |
// parent node, the packed rank tuple k (two words; smaller is better when
// score and depth tie) and the parent's score ps (for the next sibling). The
// score itself is recovered exactly from hi. Comparisons are branch-free.
// ---------------------------------------------------------------------------
struct FEntry {
  uint32_t hi, aux;
  uint64_t k;
  float ps;
};

__device__ __forceinline__ bool fbetter(const FEntry& a, const FEntry& b) {
  const uint32_t da = a.aux >> 24, db = b.aux >> 24;
  return (a.hi > b.hi) | ((a.hi == b.hi) & ((da > db) | ((da == db) & (a.k < b.k))));
}

__device__ __forceinline__ uint32_t score_key(float sc) { return ~__float_as_uint(__fadd_rn(sc, 0.0f)); }
__device__ __forceinline__ float key_score(uint32_t hi) { return __uint_as_float(~hi); }

__device__ __forceinline__ FEntry fshfl(const FEntry& e, int src) {
  FEntry o;
  o.hi = __shfl_sync(DDT_FULL_MASK, e.hi, src);
  o.aux = __shfl_sync(DDT_FULL_MASK, e.aux, src);
  o.k = __shfl_sync(DDT_FULL_MASK, e.k, src);
  o.ps = __shfl_sync(DDT_FULL_MASK, e.ps, src);
  return o;
}

__device__ __forceinline__ FEntry fsel(bool c, const FEntry& a, const FEntry& b) {
  FEntry o;
  o.hi = c ? a.hi : b.hi;
  o.aux = c ? a.aux : b.aux;
  o.k = c ? a.k : b.k;
  o.ps = c ? a.ps : b.ps;
  return o;
}

template <int SPL>
__global__ void __launch_bounds__(32) build_tree_sorted_kernel(BuildParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  pdl_wait();
  pdl_launch_dependents();
  const int b = blockIdx.x;
  const int lane = threadIdx.x;
  const int N = p.N, D = p.D, K = p.K, W = p.W, bpl = p.bpl;
  int32_t* n_parent = reinterpret_cast<int32_t*>(smem_raw);
  int32_t* n_dr = n_parent + N;  // depth << 8 | last rank
  float* n_sc = reinterpret_cast<float*>(n_dr + N);
  float* lp = n_sc + N;
  int32_t* tk = reinterpret_cast<int32_t*>(lp + D * K);
  const int L = p.cache_len[b];
  const int root = p.root_tok[b];
  const bool bad = load_drafter(p, b, lp, tk, lane);

  int32_t* o_tok = p.node_tok + (size_t)b * N;
  int32_t* o_par = p.parent + (size_t)b * N;
  int32_t* o_dep = p.depth + (size_t)b * N;
  int32_t* o_pos = p.pos + (size_t)b * N;
  float* o_sc = p.score + (size_t)b * N;
  uint32_t* o_mask = p.mask + (size_t)b * N * W;

  int n = 0;
  if (!bad) {
    FEntry fr[SPL];
#pragma unroll
    for (int q = 0; q < SPL; ++q) fr[q] = FEntry{0u, 0u, 0ull, 0.0f};
    if (lane == 0) {
      fr[0].hi = score_key(__fadd_rn(0.0f, lp[0]));  // rank 0 at depth 1, parent = root
      fr[0].aux = (127u - 1u) << 24;
      n_parent[0] = -1;
      n_dr[0] = 0;
      n_sc[0] = 0.0f;
    }
    int fsize = (N > 1) ? 1 : 0;
    n = 1;
    while (n < N && fsize > 0) {
      // pop entry 0 (lane 0, register 0)
      const FEntry w = fshfl(fr[0], 0);
      const int wd = 127 - static_cast<int>(w.aux >> 24);
      const int wr = static_cast<int>((w.aux >> 16) & 0xffu), wpar = static_cast<int>(w.aux & 0xffffu);
      const float wsc = key_score(w.hi);
      const int i = n;
      // successors: first child (rank 0 one level down) and next sibling
      const bool has_c = wd < D, has_s = wr + 1 < K;
      const float lc = lp[has_c ? wd * K : 0];
      const float ls = lp[has_s ? (wd - 1) * K + wr + 1 : 0];
      const FEntry c{score_key(__fadd_rn(wsc, lc)), ((uint32_t)(126 - wd) << 24) | (uint32_t)i, w.k << bpl, wsc};
      const FEntry sb{score_key(__fadd_rn(w.ps, ls)), w.aux + 0x10000u, w.k + 1ull, w.ps};
      // node record: warp-uniform values stored by every lane (one wavefront
      // each, no divergent branch)
      n_parent[i] = wpar;
      n_dr[i] = (wd << 8) | wr;
      n_sc[i] = wsc;
      const int ns = (int)has_c + (int)has_s;
      const bool c_first = has_c & (!has_s | fbetter(c, sb));
      const FEntry s0 = fsel(c_first, c, sb);
      const FEntry s1 = fsel(c_first, sb, c);
      // ranks of the successors among the remaining entries (old 1 .. fsize-1)
      int p0 = 0, p1 = 0;
#pragma unroll
      for (int q = 0; q < SPL; ++q) {
        const int f = 32 * q + lane;
        const bool valid = (f >= 1) & (f < fsize);
        p0 += __popc(__ballot_sync(DDT_FULL_MASK, valid & fbetter(fr[q], s0)));
        p1 += __popc(__ballot_sync(DDT_FULL_MASK, valid & fbetter(fr[q], s1)));
      }
      if (ns == 0) p0 = 32 * SPL;  // every entry moves up by one
      // merge: new entry f comes from old f + 1 (f < p0), s0 (f == p0), old f
      // (between the successors), s1 (f == p1 + 1) or old f - 1 (after both)
      FEntry nf[SPL];
#pragma unroll
      for (int q = 0; q < SPL; ++q) {
        const int f = 32 * q + lane;
        const int delta = 1 - (f > p0 ? 1 : 0) - ((ns == 2 && f > p1 + 1) ? 1 : 0);
        const int src = (lane + delta) & 31;
        FEntry v = fshfl(fr[q], src);
        if (q + 1 < SPL) {  // lane 31 moving up reads lane 0 of the next register
          const FEntry t = fshfl(fr[q + 1 < SPL ? q + 1 : q], src);
          v = fsel(lane == 31 && delta == 1, t, v);
        }
        if (q > 0) {  // lane 0 moving down reads lane 31 of the previous register
          const FEntry t = fshfl(fr[q > 0 ? q - 1 : q], src);
          v = fsel(lane == 0 && delta == -1, t, v);
        }
        v = fsel(f == p0, s0, v);
        v = fsel(ns == 2 && f == p1 + 1, s1, v);
        nf[q] = v;
      }
#pragma unroll
      for (int q = 0; q < SPL; ++q) fr[q] = nf[q];
      ++n;
      // entries that can still be popped: N - n more pops at most
      fsize = min(min(fsize - 1 + ns, N - n), 32 * SPL);
    }
    __syncwarp();
    // outputs (coalesced) and ancestor masks
    for (int j = lane; j < n; j += 32) {
      const int dr = n_dr[j];
      const int d = dr >> 8;
      o_tok[j] = j == 0 ? root : tk[(d - 1) * K + (dr & 0xff)];
      o_par[j] = n_parent[j];
      o_dep[j] = d;
      o_pos[j] = L + d;
      o_sc[j] = n_sc[j];
    }
    write_masks(o_mask, W, n, n_parent, lane);
  }
  write_pads(o_tok, o_par, o_dep, o_pos, o_sc, o_mask, W, n, N, lane);
  if (lane == 0) {
    p.n_nodes[b] = n;
    if (p.dev_status) p.dev_status[b] = bad ? DDT_ERR_INPUT : DDT_OK;
  }
}

// ---------------------------------------------------------------------------
// Packed-key variant of the sorted frontier, used when the rank tuples of
// every entry that can exist fit 25 bits (bpl * min(D, N) <= 25, e.g. K 8 x
// D 8): the whole order is then one 64-bit integer,
//   key = score key << 32 | (127 - depth) << 25 | (2^25 - 1 - k),
// larger is better, and an entry is four words (key, rank << 16 | parent,
// parent's score). Same pop / merge as build_tree_sorted_kernel.
// ---------------------------------------------------------------------------
constexpr uint32_t kKMask = (1u << 25) - 1u;

struct PEntry {
  uint64_t key;
  uint32_t aux;
  float ps;
};

__device__ __forceinline__ PEntry pshfl(const PEntry& e, int src) {
  PEntry o;
  o.key = __shfl_sync(DDT_FULL_MASK, e.key, src);
  o.aux = __shfl_sync(DDT_FULL_MASK, e.aux, src);
  o.ps = __shfl_sync(DDT_FULL_MASK, e.ps, src);
  return o;
}

__device__ __forceinline__ PEntry psel(bool c, const PEntry& a, const PEntry& b) {
  PEntry o;
  o.key = c ? a.key : b.key;
  o.aux = c ? a.aux : b.aux;
  o.ps = c ? a.ps : b.ps;
  return o;
}

__device__ __forceinline__ uint64_t packed_key(float sc, int d, uint32_t k) {
  return (static_cast<uint64_t>(score_key(sc)) << 32) | (static_cast<uint64_t>(127 - d) << 25) |
         static_cast<uint64_t>(kKMask - k);
}

template <int SPL>
__global__ void __launch_bounds__(32) build_tree_packed_kernel(BuildParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  pdl_wait();
  pdl_launch_dependents();
  const int b = blockIdx.x;
  const int lane = threadIdx.x;
  const int N = p.N, D = p.D, K = p.K, W = p.W, bpl = p.bpl;
  int32_t* n_parent = reinterpret_cast<int32_t*>(smem_raw);
  int32_t* n_dr = n_parent + N;  // depth << 8 | last rank
  float* n_sc = reinterpret_cast<float*>(n_dr + N);
  float* lp = n_sc + N;
  int32_t* tk = reinterpret_cast<int32_t*>(lp + D * K);
  const int L = p.cache_len[b];
  const int root = p.root_tok[b];
  const bool bad = load_drafter(p, b, lp, tk, lane);

  int32_t* o_tok = p.node_tok + (size_t)b * N;
  int32_t* o_par = p.parent + (size_t)b * N;
  int32_t* o_dep = p.depth + (size_t)b * N;
  int32_t* o_pos = p.pos + (size_t)b * N;
  float* o_sc = p.score + (size_t)b * N;
  uint32_t* o_mask = p.mask + (size_t)b * N * W;

  int n = 0;
  if (!bad) {
    PEntry fr[SPL];
#pragma unroll
    for (int q = 0; q < SPL; ++q) fr[q] = PEntry{0ull, 0u, 0.0f};
    if (lane == 0) {
      fr[0].key = packed_key(__fadd_rn(0.0f, lp[0]), 1, 0u);  // rank 0 at depth 1, parent = root
      n_parent[0] = -1;
      n_dr[0] = 0;
      n_sc[0] = 0.0f;
    }
    int fsize = (N > 1) ? 1 : 0;
    n = 1;
    while (n < N && fsize > 0) {
      const PEntry w = pshfl(fr[0], 0);
      const int wd = 127 - static_cast<int>((w.key >> 25) & 0x7fu);
      const uint32_t wk = kKMask - static_cast<uint32_t>(w.key & kKMask);
      const float wsc = key_score(static_cast<uint32_t>(w.key >> 32));
      const int wr = static_cast<int>(w.aux >> 16), wpar = static_cast<int>(w.aux & 0xffffu);
      const int i = n;
      const bool has_c = wd < D, has_s = wr + 1 < K;
      const float lc = lp[has_c ? wd * K : 0];
      const float ls = lp[has_s ? (wd - 1) * K + wr + 1 : 0];
      const PEntry c{packed_key(__fadd_rn(wsc, lc), wd + 1, wk << bpl), static_cast<uint32_t>(i), wsc};
      const PEntry sb{packed_key(__fadd_rn(w.ps, ls), wd, wk + 1u), w.aux + 0x10000u, w.ps};
      // node record: warp-uniform values stored by every lane (one wavefront
      // each, no divergent branch)
      n_parent[i] = wpar;
      n_dr[i] = (wd << 8) | wr;
      n_sc[i] = wsc;
      const int ns = (int)has_c + (int)has_s;
      const bool c_first = has_c & (!has_s | (c.key > sb.key));
      const PEntry s0 = psel(c_first, c, sb);
      const PEntry s1 = psel(c_first, sb, c);
      int p0 = 0, p1 = 0;
#pragma unroll
      for (int q = 0; q < SPL; ++q) {
        const int f = 32 * q + lane;
        const bool valid = (f >= 1) & (f < fsize);
        p0 += __popc(__ballot_sync(DDT_FULL_MASK, valid & (fr[q].key > s0.key)));
        p1 += __popc(__ballot_sync(DDT_FULL_MASK, valid & (fr[q].key > s1.key)));
      }
      if (ns == 0) p0 = 32 * SPL;
      PEntry nf[SPL];
#pragma unroll
      for (int q = 0; q < SPL; ++q) {
        const int f = 32 * q + lane;
        const int delta = 1 - (f > p0 ? 1 : 0) - ((ns == 2 && f > p1 + 1) ? 1 : 0);
        const int src = (lane + delta) & 31;
        PEntry v = pshfl(fr[q], src);
        if (q + 1 < SPL) {
          const PEntry t = pshfl(fr[q + 1 < SPL ? q + 1 : q], src);
          v = psel(lane == 31 && delta == 1, t, v);
        }
        if (q > 0) {
          const PEntry t = pshfl(fr[q > 0 ? q - 1 : q], src);
          v = psel(lane == 0 && delta == -1, t, v);
        }
        v = psel(f == p0, s0, v);
        v = psel(ns == 2 && f == p1 + 1, s1, v);
        nf[q] = v;
      }
#pragma unroll
      for (int q = 0; q < SPL; ++q) fr[q] = nf[q];
      ++n;
      fsize = min(min(fsize - 1 + ns, N - n), 32 * SPL);
    }
    __syncwarp();
    for (int j = lane; j < n; j += 32) {
      const int dr = n_dr[j];
      const int d = dr >> 8;
      o_tok[j] = j == 0 ? root : tk[(d - 1) * K + (dr & 0xff)];
      o_par[j] = n_parent[j];
      o_dep[j] = d;
      o_pos[j] = L + d;
      o_sc[j] = n_sc[j];
    }
    write_masks(o_mask, W, n, n_parent, lane);
  }
  write_pads(o_tok, o_par, o_dep, o_pos, o_sc, o_mask, W, n, N, lane);
  if (lane == 0) {
    p.n_nodes[b] = n;
    if (p.dev_status) p.dev_status[b] = bad ? DDT_ERR_INPUT : DDT_OK;
  }
}

template <int SPL>
static int launch_packed(const BuildParams& p, cudaStream_t stream) {
  const size_t smem = (size_t)p.N * 12 + (size_t)p.D * p.K * 8;
  if (smem > 48 * 1024) {
    if (cudaFuncSetAttribute(build_tree_packed_kernel<SPL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return DDT_ERR_CUDA;
  }
  return launch_pdl(build_tree_packed_kernel<SPL>, (unsigned)p.B, 32, smem, stream, p);
}

template <int SPL>
static int launch_sorted(const BuildParams& p, cudaStream_t stream) {
  const size_t smem = (size_t)p.N * 12 + (size_t)p.D * p.K * 8;
  if (smem > 48 * 1024) {
    if (cudaFuncSetAttribute(build_tree_sorted_kernel<SPL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return DDT_ERR_CUDA;
  }
  return launch_pdl(build_tree_sorted_kernel<SPL>, (unsigned)p.B, 32, smem, stream, p);
}

int launch_build_tree(const BuildParams& p, cudaStream_t stream) {
  // every entry that can exist has depth <= min(D, N): its rank tuple needs
  // bpl bits per level
  const bool packed = (long long)p.bpl * (p.D < p.N ? p.D : p.N) <= 25;
  if (packed && p.N <= 64) return launch_packed<1>(p, stream);
  if (packed && p.N <= 128) return launch_packed<2>(p, stream);
  if (packed && p.N <= 256) return launch_packed<4>(p, stream);
  if (p.N <= 64) return launch_sorted<1>(p, stream);
  if (p.N <= 128) return launch_sorted<2>(p, stream);
  if (p.N <= 256) return launch_sorted<4>(p, stream);
  const size_t smem = build_smem_bytes(p.N, p.D, p.K);
  if (smem > 48 * 1024) {
    if (cudaFuncSetAttribute(build_tree_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return DDT_ERR_CUDA;
  }
  return launch_pdl(build_tree_kernel, (unsigned)p.B, 32, smem, stream, p);
}

}  // namespace ddt
