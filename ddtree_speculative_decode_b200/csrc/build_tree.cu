// Best-first draft-tree build: one warp per request, or one CTA per request
// for wide, shallow trees (the level-synchronous build further down).
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
#include <mutex>

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

// ---------------------------------------------------------------------------
// Level-synchronous build for shallow, wide trees (one CTA of 512 threads per
// request). With M = N - 1 paths wanted, let list_d be the best M paths of
// depth d in (score desc, rank tuple asc) order among the children of
// list_{d-1} (list_0 = the root). The first M paths of the whole order are
// the best M of the union of the lists: a depth-d path left out of list_d
// has M better paths of its own depth, and a path whose prefix was left out
// ranks after that prefix, which already has M better paths. Each level's
// best M (and finally the union's) are found by a radix select over the
// packed order key (inverted score key, depth, rank tuple), one byte per
// pass, most significant first, with shared-memory histograms; the final M
// are then placed by their ranks among one another, so node i is the i-th
// path of the best-first search's pops.
// ---------------------------------------------------------------------------
constexpr int kLvThreads = 512;
constexpr int kLvMaxN = 256;     // M <= 255 entries per level
constexpr int kLvMaxD = 16;
constexpr int kLvMaxP = 4096;    // candidates of a level (at most 255 x 16) or the union (16 x 255)

struct LvCand {
  uint32_t hi;   // ~order key of the score: smaller is better
  uint32_t tag;  // depth << 16 | index (index = parent entry * K + rank, or entry of its level)
  uint64_t k;    // packed rank tuple: smaller is lexicographically first
};

__device__ __forceinline__ bool lv_less(const LvCand& a, const LvCand& b) {
  if (a.hi != b.hi) return a.hi < b.hi;
  if ((a.tag >> 16) != (b.tag >> 16)) return (a.tag >> 16) < (b.tag >> 16);
  return a.k < b.k;
}

struct LvSmem {
  LvCand cand[kLvMaxP];
  LvCand order[kLvMaxN];             // the union's first M, then in order
  float sc[kLvMaxD][kLvMaxN];
  uint64_t key[kLvMaxD][kLvMaxN];
  int16_t par[kLvMaxD][kLvMaxN];     // entry of the level above (-1: the root)
  uint8_t rk[kLvMaxD][kLvMaxN];      // last rank
  int16_t node[kLvMaxD][kLvMaxN];    // node index, or 0 when not among the first M
  int32_t n_parent[kLvMaxN];
  float lp[kLvMaxD * 32];
  int32_t tk[kLvMaxD * 32];
  int cnt[kLvMaxD + 1];
  int hist[kLvThreads / 32][256];   // one histogram per warp (no contention between warps)
  uint32_t lo_hi, hi_hi;             // smallest and largest hi of the candidates
  uint32_t t_hi, t_dep;              // radix select: threshold's decided bits
  uint64_t t_k;
  int sel_digit, sel_rank, sel_full;
  int wsum[kLvThreads / 32];
  int bad;
};

__device__ __forceinline__ uint32_t lv_hi(float sc) { return ~float_order_key(sc); }
__device__ __forceinline__ float lv_score(uint32_t hi) {
  const uint32_t u = ~hi;
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}

// Radix select over S.cand[0, P): after it, a candidate is among the `want`
// smallest keys iff lv_in(...) holds. Key bits, most significant first: hi
// (32), depth (8, only when `depth`), k (64); one byte per pass. Passes stop
// once every candidate sharing the decided prefix is taken.
struct LvSel {
  uint32_t m_hi, m_dep;  // decided bits
  uint64_t m_k;
};

__device__ __forceinline__ bool lv_match(const LvSmem& S, const LvSel& m, const LvCand& c) {
  return ((c.hi ^ S.t_hi) & m.m_hi) == 0u && (((c.tag >> 16) ^ S.t_dep) & m.m_dep) == 0u &&
         ((c.k ^ S.t_k) & m.m_k) == 0ull;
}

// taken: the decided bits of the key are at most the threshold's
__device__ __forceinline__ bool lv_in(const LvSmem& S, const LvSel& m, const LvCand& c) {
  const uint32_t a = c.hi & m.m_hi, ta = S.t_hi & m.m_hi;
  if (a != ta) return a < ta;
  const uint32_t d = (c.tag >> 16) & m.m_dep, td = S.t_dep & m.m_dep;
  if (d != td) return d < td;
  return (c.k & m.m_k) <= (S.t_k & m.m_k);
}

// Exclusive offset of this thread's count among the CTA's threads (thread
// order), and the total; the whole CTA calls it.
__device__ __forceinline__ int lv_offset(LvSmem& S, int count, int& total) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int incl = count;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(DDT_FULL_MASK, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) S.wsum[warp] = incl;
  __syncthreads();
  int base = 0;
  total = 0;
  for (int w = 0; w < kLvThreads / 32; ++w) {
    const int v = S.wsum[w];
    if (w < warp) base += v;
    total += v;
  }
  __syncthreads();
  return base + incl - count;
}

// Radix select over S.cand[0, P): afterwards a candidate is among the `want`
// smallest keys iff lv_in holds. The key, most significant first: hi (32
// bits), depth (8, only when `depth`), k (kbits: the rank tuples' width).
// Each pass histograms the next window of up to 8 undecided bits of the
// candidates that match the decided prefix; hi's windows start at the first
// bit where the candidates' scores differ. Passes stop once every candidate
// sharing the decided prefix is taken (keys are distinct).
__device__ LvSel lv_select(LvSmem& S, int P, int want, bool depth, int kbits) {
  LvSel m{0u, 0u, 0ull};
  const int tid = threadIdx.x;
  if (tid == 0) {
    S.t_hi = 0u;
    S.t_dep = 0u;
    S.t_k = 0ull;
    S.lo_hi = 0xffffffffu;
    S.hi_hi = 0u;
  }
  __syncthreads();
  if (want >= P) return m;  // every candidate is taken
  {
    uint32_t lo = 0xffffffffu, hi = 0u;
    for (int i = tid; i < P; i += kLvThreads) {
      const uint32_t v = S.cand[i].hi;
      lo = min(lo, v);
      hi = max(hi, v);
    }
    lo = __reduce_min_sync(DDT_FULL_MASK, lo);
    hi = __reduce_max_sync(DDT_FULL_MASK, hi);
    if ((tid & 31) == 0) {
      atomicMin(&S.lo_hi, lo);
      atomicMax(&S.hi_hi, hi);
    }
  }
  __syncthreads();
  const uint32_t diff = S.lo_hi ^ S.hi_hi;
  int hi_top = diff ? 31 - __clz(diff) : -1;  // highest undecided bit of hi (the bits above agree)
  m.m_hi = hi_top < 0 ? 0xffffffffu : (hi_top >= 31 ? 0u : ~((2u << hi_top) - 1u));
  const uint32_t t_hi0 = S.lo_hi & m.m_hi;
  __syncthreads();
  if (tid == 0) S.t_hi = t_hi0;
  bool dep_left = depth;
  int k_top = kbits - 1;
  __syncthreads();
  int rank = want;  // how many of the candidates matching the prefix are still to take
  for (;;) {
    int field, lo, width;
    if (hi_top >= 0) {
      field = 0;
      lo = hi_top >= 7 ? hi_top - 7 : 0;
      width = hi_top - lo + 1;
    } else if (dep_left) {
      field = 1;
      lo = 0;
      width = 8;
    } else if (k_top >= 0) {
      field = 2;
      lo = k_top >= 7 ? k_top - 7 : 0;
      width = k_top - lo + 1;
    } else {
      break;  // every bit decided
    }
    const uint32_t wmask = (1u << width) - 1u;
    const int warp = tid >> 5;
    for (int i = tid; i < (kLvThreads / 32) * 256; i += kLvThreads) (&S.hist[0][0])[i] = 0;
    __syncthreads();
    for (int i = tid; i < P; i += kLvThreads) {
      const LvCand c = S.cand[i];
      if (!lv_match(S, m, c)) continue;
      const uint32_t v = field == 0 ? c.hi >> lo : field == 1 ? (c.tag >> 16) : (uint32_t)(c.k >> lo);
      atomicAdd(&S.hist[warp][v & wmask], 1);  // this warp's own histogram
    }
    __syncthreads();
    if (tid < 32) {
      // bins 8 lane .. 8 lane + 7 summed over the warps: the bin where the
      // running count reaches rank
      const int lane = tid;
      int h[8], sum = 0;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        int v = 0;
#pragma unroll
        for (int w = 0; w < kLvThreads / 32; ++w) v += S.hist[w][8 * lane + t];
        h[t] = v;
        sum += v;
      }
      int incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(DDT_FULL_MASK, incl, o);
        if (lane >= o) incl += v;
      }
      int before = incl - sum;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        if (before < rank && rank <= before + h[t]) {
          S.sel_digit = 8 * lane + t;
          S.sel_rank = rank - before;
          S.sel_full = (h[t] == rank - before) ? 1 : 0;
        }
        before += h[t];
      }
    }
    __syncthreads();
    const uint32_t dg = (uint32_t)S.sel_digit;
    rank = S.sel_rank;
    const bool full = S.sel_full != 0;
    if (field == 0) {
      m.m_hi |= wmask << lo;
      if (tid == 0) S.t_hi |= dg << lo;
      hi_top = lo - 1;
    } else if (field == 1) {
      m.m_dep |= 0xffu;
      if (tid == 0) S.t_dep |= dg;
      dep_left = false;
    } else {
      m.m_k |= (uint64_t)wmask << lo;
      if (tid == 0) S.t_k |= (uint64_t)dg << lo;
      k_top = lo - 1;
    }
    __syncthreads();
    if (full) break;
  }
  return m;
}

__global__ void __launch_bounds__(kLvThreads) build_tree_level_kernel(BuildParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  LvSmem& S = *reinterpret_cast<LvSmem*>(smem_raw);
  pdl_wait();
  pdl_launch_dependents();
  const int b = blockIdx.x, tid = threadIdx.x;
  const int N = p.N, D = p.D, K = p.K, W = p.W, bpl = p.bpl;
  const int M = N - 1;
  const int L = p.cache_len[b];
  const int root = p.root_tok[b];
  if (tid < 32) {
    const bool bad = load_drafter(p, b, S.lp, S.tk, tid);
    if (tid == 0) S.bad = bad ? 1 : 0;
  }
  __syncthreads();
  const bool bad = S.bad != 0;
  int32_t* o_tok = p.node_tok + (size_t)b * N;
  int32_t* o_par = p.parent + (size_t)b * N;
  int32_t* o_dep = p.depth + (size_t)b * N;
  int32_t* o_pos = p.pos + (size_t)b * N;
  float* o_sc = p.score + (size_t)b * N;
  uint32_t* o_mask = p.mask + (size_t)b * N * W;
  int n = 0;
  if (!bad) {
    // levels: list_d = the best M children of list_{d-1}
    int prev = 1;  // list_0: the root
    int total = 0;
    for (int d = 1; d <= D && M > 0; ++d) {
      const int P = prev * K;
      for (int i = tid; i < P; i += kLvThreads) {
        const int j = i / K, r = i - j * K;
        const float ps = d == 1 ? 0.0f : S.sc[d - 2][j];
        const uint64_t pk = d == 1 ? 0ull : S.key[d - 2][j];
        LvCand c;
        c.hi = lv_hi(__fadd_rn(ps, S.lp[(d - 1) * K + r]));
        c.tag = (uint32_t)i;  // depth 0 here: every candidate of the level has the same one
        c.k = (pk << bpl) | (uint64_t)r;
        S.cand[i] = c;
      }
      __syncthreads();
      const int cnt = P < M ? P : M;
      const LvSel m = lv_select(S, P, cnt, false, bpl * d);
      {
        // the taken candidates, in thread order, at offsets from a block scan
        int mine = 0;
        for (int i = tid; i < P; i += kLvThreads) mine += lv_in(S, m, S.cand[i]) ? 1 : 0;
        int tot = 0;
        int e = lv_offset(S, mine, tot);
        for (int i = tid; i < P; i += kLvThreads) {
          const LvCand c = S.cand[i];
          if (!lv_in(S, m, c)) continue;
          if (e < kLvMaxN) {  // exactly cnt are taken (keys are distinct)
            const int ci = (int)(c.tag & 0xffffu);
            const int j = ci / K, r = ci - j * K;
            S.sc[d - 1][e] = lv_score(c.hi);
            S.key[d - 1][e] = c.k;
            S.par[d - 1][e] = (int16_t)(d == 1 ? -1 : j);
            S.rk[d - 1][e] = (uint8_t)r;
          }
          ++e;
        }
      }
      if (tid == 0) S.cnt[d] = cnt;
      __syncthreads();
      prev = cnt;
      total += cnt;
    }
    // the union's best M, then their order by ranks among one another
    const int levels = total > 0 ? D : 0;
    for (int i = tid; i < total; i += kLvThreads) {
      int d = 1, e = i;
      while (d <= levels && e >= S.cnt[d]) {
        e -= S.cnt[d];
        ++d;
      }
      LvCand c;
      c.hi = lv_hi(S.sc[d - 1][e]);
      c.tag = ((uint32_t)d << 16) | (uint32_t)e;
      c.k = S.key[d - 1][e];
      S.cand[i] = c;
    }
    for (int i = tid; i < kLvMaxD * kLvMaxN; i += kLvThreads) (&S.node[0][0])[i] = 0;
    __syncthreads();
    const int sel = total < M ? total : M;
    if (sel > 0) {
      const LvSel m = lv_select(S, total, sel, true, bpl * D);
      {
        int mine = 0;
        for (int i = tid; i < total; i += kLvThreads) mine += lv_in(S, m, S.cand[i]) ? 1 : 0;
        int tot = 0;
        int q = lv_offset(S, mine, tot);
        for (int i = tid; i < total; i += kLvThreads) {
          const LvCand c = S.cand[i];
          if (!lv_in(S, m, c)) continue;
          if (q < kLvMaxN) S.order[q] = c;  // exactly sel are taken
          ++q;
        }
      }
      __syncthreads();
      // rank of each taken path among the others: two threads per path, each
      // counting over half of them
      LvCand mine;
      int rank = 0;
      const int me = tid >> 1, half = tid & 1;
      if (me < sel) {
        mine = S.order[me];
        const int u0 = half ? sel / 2 : 0, u1 = half ? sel : sel / 2;
#pragma unroll 4
        for (int u = u0; u < u1; ++u) rank += lv_less(S.order[u], mine) ? 1 : 0;
      }
      rank += __shfl_xor_sync(DDT_FULL_MASK, rank, 1);
      __syncthreads();
      if (me < sel && half == 0) {
        S.cand[rank] = mine;
        S.node[(mine.tag >> 16) - 1][mine.tag & 0xffffu] = (int16_t)(rank + 1);
      }
      __syncthreads();
    }
    n = 1 + sel;
    // outputs: node 0 the root, node q + 1 the q-th path
    for (int i = tid; i < n; i += kLvThreads) {
      if (i == 0) {
        o_tok[0] = root;
        o_par[0] = -1;
        o_dep[0] = 0;
        o_pos[0] = L;
        o_sc[0] = 0.0f;
        S.n_parent[0] = -1;
      } else {
        const uint32_t tag = S.cand[i - 1].tag;
        const int d = (int)(tag >> 16), e = (int)(tag & 0xffffu);
        const int pe = S.par[d - 1][e];
        const int pn = d == 1 ? 0 : (int)S.node[d - 2][pe];
        o_tok[i] = S.tk[(d - 1) * K + S.rk[d - 1][e]];
        o_par[i] = pn;
        o_dep[i] = d;
        o_pos[i] = L + d;
        o_sc[i] = S.sc[d - 1][e];
        S.n_parent[i] = pn;
      }
    }
    __syncthreads();
    // ancestor masks: one thread per node walks its parent chain (parent < child)
    for (int i = tid; i < n; i += kLvThreads) {
      uint32_t mk[kLvMaxN / 32];
#pragma unroll
      for (int w = 0; w < kLvMaxN / 32; ++w) mk[w] = 0u;
      for (int j = i; j >= 0; j = S.n_parent[j]) {
#pragma unroll
        for (int w = 0; w < kLvMaxN / 32; ++w)
          if ((j >> 5) == w) mk[w] |= 1u << (j & 31);
      }
      uint32_t* row = o_mask + (size_t)i * W;
      for (int w = 0; w < W; ++w) row[w] = w < kLvMaxN / 32 ? mk[w] : 0u;
    }
  }
  // pad rows [n, N)
  for (int i = n + tid; i < N; i += kLvThreads) {
    o_tok[i] = -1;
    o_par[i] = -1;
    o_dep[i] = -1;
    o_pos[i] = -1;
    o_sc[i] = -INFINITY;
    uint32_t* row = o_mask + (size_t)i * W;
    for (int w = 0; w < W; ++w) row[w] = 0u;
  }
  if (tid == 0) {
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

// The level build's shared-memory opt-in, set once per device (the attribute
// applies to the device current when it is set).
static bool level_build_ready() {
  static std::mutex mu;
  static int done[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lock(mu);
  if (done[dev] == 0) {
    const cudaError_t e = cudaFuncSetAttribute(build_tree_level_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)sizeof(LvSmem));
    done[dev] = e == cudaSuccess ? 1 : -1;
    if (e != cudaSuccess) (void)cudaGetLastError();
  }
  return done[dev] == 1;
}

// The level build pays D sorts of up to (N - 1) x K candidates; the warp
// build pays N - 1 pops whose cost grows with the frontier it keeps sorted.
static bool use_level_build(const BuildParams& p) {
  return p.N > 128 && p.N <= kLvMaxN && p.D <= kLvMaxD && p.K <= 16;
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
  if (use_level_build(p)) {
    if (!level_build_ready()) return DDT_ERR_CUDA;
    return launch_pdl(build_tree_level_kernel, (unsigned)p.B, kLvThreads, sizeof(LvSmem), stream, p);
  }
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
