// Drafter proposals: per row (one request's depth), the log-softmax of the
// drafter's logits over the vocabulary and its K best tokens, best first --
// the input the best-first tree build consumes.
//
// What it computes is fixed in ddt.h (ddt_drafter_topk)
// ("ddtree_speculative_decode_test_capstone", section "The Oracle Drafter":
// per-depth log-probabilities and token ids of the drafter's candidates,
// sorted best first; "autoregressive_test_driver_kdtree_engine", section "The
// Broader Context": the draft tree is built from the drafter's per-depth
// top-k).
//
// A row is split over the CTAs of one cluster (up to 8); each streams its
// slice once with 16-byte loads, a round of eight per thread in flight while
// the round before is processed. Each thread keeps a running (max, sum of
// exponentials) for the log-sum-exp; each warp keeps a sorted list of its K
// best packed keys (order-preserving value bits << 32 | ~index, so a larger
// key is a larger value or, on equal values, a lower index). Aligned rows:
// after the first round the CTA takes the K-th largest of its threads'
// maxima (a bisection over order keys, one block-wide count per bit): at
// least K of its values reach it, so no value below can be among the K
// best, and from then on a vector costs its log-sum-exp terms, a packed
// maximum and one warp vote unless its largest value reaches the threshold
// (the larger of that bound, the warp's K-th best and the best K-th entry
// any warp of the CTA has published). The few vectors that do are keyed one
// value at a time; a warp's hits are taken by one out-of-line routine,
// inserted one by one or, when many lanes hit at once, by a bitonic sort of
// the hits and a bitonic merge with the list. Unaligned rows take every
// value through that key path. One warp per CTA merges the warps' lists by
// K rounds of a warp-wide maximum, and the cluster's first CTA merges the
// CTAs' lists, read through distributed shared memory, the same way.
#include <algorithm>

#include "ddt_kernels.cuh"
#include "sm100_ptx.cuh"

namespace ddt {

using sm100::cluster_ctarank;
using sm100::cluster_sync;
using sm100::map_to_rank;
using sm100::smem_u32;

// loads from shared memory of a CTA of the cluster (address from map_to_rank)
__device__ __forceinline__ unsigned long long ld_cluster_u64(uint32_t addr) {
  unsigned long long v;
  asm volatile("ld.shared::cluster.u64 %0, [%1];" : "=l"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ float ld_cluster_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ int ld_cluster_s32(uint32_t addr) {
  int v;
  asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

constexpr int kDrThreads = 512;
constexpr int kDrWarps = kDrThreads / 32;

__device__ __forceinline__ unsigned long long drafter_key(float v, int idx) {
  return (static_cast<unsigned long long>(float_order_key(v)) << 32) |
         static_cast<unsigned long long>(~static_cast<uint32_t>(idx));
}

__device__ __forceinline__ float key_value(unsigned long long k) {
  const uint32_t u = static_cast<uint32_t>(k >> 32);
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}

constexpr float kLog2e = 1.4426950408889634f;

// 2^x by the hardware approximation (relative error about 2^-22; subnormal
// results flushed to zero)
__device__ __forceinline__ float ex2_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// log-sum-exp state in base 2: m = running max of x log2(e), s = sum of
// 2^(x log2(e) - m)
__device__ __forceinline__ void lse_merge(float& m, float& s, float m2, float s2) {
  const float M = fmaxf(m, m2);
  if (M == -INFINITY) return;
  s = (m == -INFINITY ? 0.0f : s * ex2_ftz(m - M)) + (m2 == -INFINITY ? 0.0f : s2 * ex2_ftz(m2 - M));
  m = M;
}

// Bitonic network over the warp's 32 lanes, one key per lane: the full sort
// leaves lane 0 with the largest key; the merge sorts a bitonic sequence.
__device__ __forceinline__ unsigned long long warp_sort_desc(unsigned long long x, int lane) {
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      const unsigned long long y = __shfl_xor_sync(DDT_FULL_MASK, x, j);
      // blocks of k lanes alternate direction; the lower lane of a pair keeps
      // the larger key in a descending block
      const bool keep_max = ((lane & j) == 0) == ((lane & k) == 0);
      x = keep_max ? (y > x ? y : x) : (y < x ? y : x);
    }
  }
  return x;
}

__device__ __forceinline__ unsigned long long warp_merge_desc(unsigned long long x, int lane) {
#pragma unroll
  for (int j = 16; j > 0; j >>= 1) {
    const unsigned long long y = __shfl_xor_sync(DDT_FULL_MASK, x, j);
    x = ((lane & j) == 0) ? (y > x ? y : x) : (y < x ? y : x);
  }
  return x;
}

constexpr int kMergeHits = 6;  // from this many hits one sort-merge beats serial inserts

// Takes a warp's hits (cand on the lanes set in hits, 0 elsewhere) into its
// sorted list wl (lane j = entry j, 0 = empty, lanes >= K hold 0); returns the
// new list. Out of line: one copy of the code serves every call site.
__device__ __noinline__ unsigned long long take_hits(unsigned long long wl, unsigned long long cand,
                                                     unsigned hits, int K, int lane) {
  if (__popc(hits) >= kMergeHits) {
    // sorted hits reversed (ascending) against the descending list: the
    // lane-wise maximum holds the 32 best of both as a bitonic sequence
    const unsigned long long c = warp_sort_desc(cand, lane);
    const unsigned long long crev = __shfl_sync(DDT_FULL_MASK, c, 31 - lane);
    const unsigned long long m = warp_merge_desc(wl > crev ? wl : crev, lane);
    return lane < K ? m : 0ull;
  }
  unsigned long long last = __shfl_sync(DDT_FULL_MASK, wl, K - 1);
  while (hits) {  // warp-uniform
    const int src = __ffs(hits) - 1;
    hits &= hits - 1u;
    const unsigned long long kk = __shfl_sync(DDT_FULL_MASK, cand, src);
    if (kk > last) {
      // lanes whose entry beats kk keep their place; the rest move down one
      const int pos = __popc(__ballot_sync(DDT_FULL_MASK, lane < K && wl > kk));
      const unsigned long long up = __shfl_up_sync(DDT_FULL_MASK, wl, 1);
      if (lane > pos && lane < K) wl = up;
      if (lane == pos && pos < K) wl = kk;
      last = __shfl_sync(DDT_FULL_MASK, wl, K - 1);
    }
  }
  return wl;
}

// The warp's K best keys over the lanes' sorted lists (each consumed from its
// head); round j's key ends up in lane j. Lists are destroyed.
template <int KM>
__device__ __forceinline__ unsigned long long warp_topk(unsigned long long (&k)[KM], int K, int lane) {
  unsigned long long mine = 0ull;
  for (int j = 0; j < K; ++j) {
    unsigned long long best = k[0];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long other = __shfl_xor_sync(DDT_FULL_MASK, best, o);
      best = other > best ? other : best;
    }
    if (lane == j) mine = best;
    const bool pop = best != 0ull && k[0] == best;  // keys are unique: one lane pops
#pragma unroll
    for (int i = 0; i < KM - 1; ++i) k[i] = pop ? k[i + 1] : k[i];
    if (pop) k[KM - 1] = 0ull;
  }
  return mine;
}

template <int KM, bool kBF16>
__global__ void __launch_bounds__(kDrThreads) drafter_topk_kernel(DrafterParams p) {
  pdl_wait();
  pdl_launch_dependents();
  const uint32_t crank = cluster_ctarank();  // this CTA's slice of the row
  const int r = (int)(blockIdx.x / (unsigned)p.C);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int V = p.V;
  const int v0 = min(V, (int)crank * p.chunk), v1 = min(V, v0 + p.chunk);
  const size_t esz = kBF16 ? 2 : 4;
  const unsigned char* row = static_cast<const unsigned char*>(p.logits) + (size_t)r * V * esz;

  // The warp's K best so far, lane j holding entry j (0 = empty; every
  // finite value's key is larger); wthr = its last entry, s_thr = the largest
  // last entry any warp of this CTA has published. A key at or below either
  // has K larger keys in the row, so it is dropped: after the first few
  // batches a value costs one compare and its warp one ballot.
  __shared__ unsigned long long s_thr;
  if (tid == 0) s_thr = 0ull;
  __syncthreads();
  // lo: a key just below the K-th largest of the warp's lanes' maxima over
  // the first loads (those K keys are distinct values of the row, so no key
  // below lo can be among the row's K best); it keeps the first batches,
  // where the lists are still empty, from taking every value as a hit
  unsigned long long wl = 0ull, wthr = 0ull, thr = 0ull, pub = 0ull, lo = 0ull;
  float m = -INFINITY, s = 0.0f;
  bool bad = false;
  // before each batch: the CTA's threshold; after it: publish this warp's
  auto refresh = [&]() {
    const unsigned long long c = *reinterpret_cast<volatile unsigned long long*>(&s_thr);
    thr = c > wthr ? c : wthr;
    thr = thr > lo ? thr : lo;
  };
  auto publish = [&]() {
    const unsigned long long w = wthr > lo ? wthr : lo;
    if (w > pub) {  // warp-uniform
      if (lane == 0) atomicMax(&s_thr, w);
      pub = w;
    }
  };
  // a batch of n of this lane's values (all lanes of the warp call it together)
  auto batch = [&](const float* x, int n, int idx0) {
    float y[8];
    float bm = -INFINITY;
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      if (t < n) {
        bad |= !(fabsf(x[t]) <= 3.402823466e38f);
        y[t] = x[t] * kLog2e;
        bm = fmaxf(bm, y[t]);
      }
    }
    if (bm > m) {
      s *= ex2_ftz(m - bm);
      m = bm;
    }
    float bs = 0.0f;
#pragma unroll
    for (int t = 0; t < 8; ++t)
      if (t < n) bs += ex2_ftz(y[t] - m);
    s += bs;
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      const unsigned long long key =
          (t < n && fabsf(x[t]) <= 3.402823466e38f) ? drafter_key(x[t], idx0 + t) : 0ull;
      const bool hit = key > thr;
      const unsigned hits = __ballot_sync(DDT_FULL_MASK, hit);
      if (hits) {  // warp-uniform
        wl = take_hits(wl, hit ? key : 0ull, hits, p.K, lane);
        wthr = __shfl_sync(DDT_FULL_MASK, wl, p.K - 1);
        thr = wthr > thr ? wthr : thr;
      }
    }
  };
  if (p.vec) {  // 16-byte aligned rows: 8 bf16 or 4 f32 per load
    constexpr int kPer = kBF16 ? 8 : 4;
    const int nvec = v1 / kPer;  // the slice [v0, v1) starts on a vector
    const uint4* src = reinterpret_cast<const uint4*>(row);
    // eight 16-byte loads in flight per thread (64 KB per CTA) before any is
    // used; whole warps step together (lanes past the end take no values)
    constexpr int kU = 8;
    auto value_of = [](const uint4& r, int t) -> float {
      const uint32_t w = t < (kBF16 ? 2 : 1) ? r.x : t < (kBF16 ? 4 : 2) ? r.y : t < (kBF16 ? 6 : 3) ? r.z : r.w;
      if (!kBF16) return __uint_as_float(w);
      return __uint_as_float((t & 1) ? (w & 0xffff0000u) : (w << 16));
    };
    // largest and smallest value of a vector (pairs of bf16 folded first)
    auto vec_max_min = [](const uint4& r, float& mx, float& mn) {
      if (kBF16) {
        auto h = [](uint32_t w) { return *reinterpret_cast<const __nv_bfloat162*>(&w); };
        const __nv_bfloat162 a = __hmax2(__hmax2(h(r.x), h(r.y)), __hmax2(h(r.z), h(r.w)));
        const __nv_bfloat162 c = __hmin2(__hmin2(h(r.x), h(r.y)), __hmin2(h(r.z), h(r.w)));
        mx = fmaxf(__low2float(a), __high2float(a));
        mn = fminf(__low2float(c), __high2float(c));
      } else {
        mx = fmaxf(fmaxf(__uint_as_float(r.x), __uint_as_float(r.y)), fmaxf(__uint_as_float(r.z), __uint_as_float(r.w)));
        mn = fminf(fminf(__uint_as_float(r.x), __uint_as_float(r.y)), fminf(__uint_as_float(r.z), __uint_as_float(r.w)));
      }
    };
    // One round of kU vectors per lane: the log-sum-exp over every value,
    // then the keys of the vectors whose largest value reaches the threshold
    // (thr's value); a vector no lane of the warp needs costs one vote.
    auto round = [&](const uint4 (&v)[kU], int e0) {
      float vmax[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int e = e0 + lane + u * kDrThreads;
        float mx, mn;
        vec_max_min(v[u], mx, mn);
        if (e >= nvec) mx = -INFINITY;
        // a non-finite value: +inf shows in the max, -inf in the min, NaN in
        // the sum of exponentials below
        if (e < nvec && !(fabsf(mx) <= 3.402823466e38f && fabsf(mn) <= 3.402823466e38f)) bad = true;
        vmax[u] = mx;
        if (e < nvec) {
          const float ym = mx * kLog2e;
          if (ym > m) {
            s *= ex2_ftz(m - ym);
            m = ym;
          }
          float bs = 0.0f;
#pragma unroll
          for (int t = 0; t < kPer; ++t) bs += ex2_ftz(fmaf(value_of(v[u], t), kLog2e, -m));
          s += bs;
        }
      }
      if (!(s == s)) bad = true;
      refresh();
      // vectors some lane of the warp may need: a vote each; then one copy of
      // the key code walks them (kept out of the unrolled path: rare, and the
      // instruction cache is what a second copy per vector would cost)
      const float tv = key_value(thr);
      unsigned need = 0u;
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int e = e0 + lane + u * kDrThreads;
        if (__any_sync(DDT_FULL_MASK, e < nvec && (thr == 0ull || vmax[u] >= tv))) need |= 1u << u;
      }
      while (need) {  // warp-uniform
        const int u = __ffs(need) - 1;
        need &= need - 1u;
        uint4 cur = v[0];
        float cmax = vmax[0];
#pragma unroll
        for (int q = 1; q < kU; ++q)
          if (q == u) {
            cur = v[q];
            cmax = vmax[q];
          }
        const int e = e0 + lane + u * kDrThreads;
        const bool maybe = e < nvec && (thr == 0ull || cmax >= key_value(thr));
#pragma unroll 1
        for (int t = 0; t < kPer; ++t) {
          const float xv = value_of(cur, t);
          const unsigned long long key =
              (maybe && fabsf(xv) <= 3.402823466e38f) ? drafter_key(xv, e * kPer + t) : 0ull;
          const bool hit = key > thr;
          const unsigned hits = __ballot_sync(DDT_FULL_MASK, hit);
          if (hits) {  // warp-uniform
            wl = take_hits(wl, hit ? key : 0ull, hits, p.K, lane);
            wthr = __shfl_sync(DDT_FULL_MASK, wl, p.K - 1);
            thr = wthr > thr ? wthr : thr;
          }
        }
      }
      publish();
    };
    // The first round of every warp (all warps take part, lanes past the end
    // with no values), then the CTA's K-th largest of its threads' maxima by
    // a bisection over order keys: at least K of the slice's values reach
    // it, so every value below it is out, and lo starts at that bound. Each
    // round's loads are issued before the round before it is processed.
    auto load = [&](uint4 (&v)[kU], int e0) {
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int e = e0 + lane + u * kDrThreads;
        v[u] = e < nvec ? __ldcs(src + e) : make_uint4(0u, 0u, 0u, 0u);
      }
    };
    int e0 = v0 / kPer + warp * 32;
    uint4 v[kU], nv[kU];
    load(v, e0);
    load(nv, e0 + kU * kDrThreads);
    {
      float tm = -INFINITY;
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int e = e0 + lane + u * kDrThreads;
        float mx, mn;
        vec_max_min(v[u], mx, mn);
        if (e < nvec && fabsf(mx) <= 3.402823466e38f) tm = fmaxf(tm, mx);
      }
      const uint32_t tk = tm > -INFINITY ? float_order_key(tm) : 0u;
      uint32_t t = 0u;
      for (int bit = 31; bit >= 0; --bit) {  // every thread of the CTA, same trips
        const uint32_t cand = t | (1u << bit);
        if (__syncthreads_count(tk >= cand) >= p.K) t = cand;
      }
      lo = t > 0u ? (static_cast<unsigned long long>(t) << 32) - 1ull : 0ull;
    }
    while (e0 < nvec) {  // warp-uniform
      const int en = e0 + kU * kDrThreads;
      round(v, e0);
#pragma unroll
      for (int u = 0; u < kU; ++u) v[u] = nv[u];
      if (en + kU * kDrThreads < nvec) load(nv, en + kU * kDrThreads);
      e0 = en;
    }
  } else {
    for (int i0 = v0 + warp * 32; i0 < v1; i0 += kDrThreads) {  // whole warps step together
      const int i = i0 + lane;
      float x[8];
      x[0] = i < v1 ? (kBF16 ? bf16_bits_to_float(reinterpret_cast<const uint16_t*>(row)[i])
                             : reinterpret_cast<const float*>(row)[i])
                    : 0.0f;
      refresh();
      batch(x, i < v1 ? 1 : 0, i);
      publish();
    }
  }
  // ---- combine: log-sum-exp and non-finite flag
  __shared__ float s_m[kDrWarps], s_s[kDrWarps];
  __shared__ int s_bad;
  __shared__ unsigned long long s_keys[kDrWarps][KM];
  if (tid == 0) s_bad = 0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(DDT_FULL_MASK, m, o), s2 = __shfl_xor_sync(DDT_FULL_MASK, s, o);
    lse_merge(m, s, m2, s2);
  }
  const bool wbad = __any_sync(DDT_FULL_MASK, bad);
  const unsigned long long wk = wl;  // this warp's K best: lane j holds entry j
  __syncthreads();
  if (lane == 0) {
    s_m[warp] = m;
    s_s[warp] = s;
    if (wbad) s_bad = 1;
  }
  if (lane < p.K) s_keys[warp][lane] = wk;
  __syncthreads();
  // this CTA's K best and (max, sum) over its warps, for the cluster's first CTA
  __shared__ unsigned long long s_cta[KM];
  __shared__ float s_cta_m, s_cta_s;
  __shared__ int s_cta_bad;
  if (warp == 0) {
    unsigned long long kk[KM];
#pragma unroll
    for (int i = 0; i < KM; ++i) kk[i] = (lane < kDrWarps && i < p.K) ? s_keys[lane][i] : 0ull;
    const unsigned long long best = warp_topk<KM>(kk, p.K, lane);
    float M = lane < kDrWarps ? s_m[lane] : -INFINITY, S = lane < kDrWarps ? s_s[lane] : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float m2 = __shfl_xor_sync(DDT_FULL_MASK, M, o), s2 = __shfl_xor_sync(DDT_FULL_MASK, S, o);
      lse_merge(M, S, m2, s2);
    }
    if (lane < p.K) s_cta[lane] = best;
    if (lane == 0) {
      s_cta_m = M;
      s_cta_s = S;
      s_cta_bad = s_bad;
    }
  }
  // every thread of every CTA of the cluster takes both cluster barriers
  cluster_sync();
  if (crank == 0 && warp == 0) {
    // lane q < C reads CTA q's list and (max, sum)
    const bool has = lane < p.C;
    unsigned long long kk[KM];
#pragma unroll
    for (int i = 0; i < KM; ++i)
      kk[i] = (has && i < p.K) ? ld_cluster_u64(map_to_rank(smem_u32(&s_cta[i]), (uint32_t)lane)) : 0ull;
    float M = has ? ld_cluster_f32(map_to_rank(smem_u32(&s_cta_m), (uint32_t)lane)) : -INFINITY;
    float S = has ? ld_cluster_f32(map_to_rank(smem_u32(&s_cta_s), (uint32_t)lane)) : 0.0f;
    const int qbad = has ? ld_cluster_s32(map_to_rank(smem_u32(&s_cta_bad), (uint32_t)lane)) : 0;
    const unsigned long long best = warp_topk<KM>(kk, p.K, lane);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float m2 = __shfl_xor_sync(DDT_FULL_MASK, M, o), s2 = __shfl_xor_sync(DDT_FULL_MASK, S, o);
      lse_merge(M, S, m2, s2);
    }
    const bool row_bad = __any_sync(DDT_FULL_MASK, qbad != 0);
    if (lane < p.K) {
      const float lse = (M + log2f(S)) * 0.6931471805599453f;
      p.logp[(size_t)r * p.K + lane] = row_bad ? -INFINITY : key_value(best) - lse;
      p.tok[(size_t)r * p.K + lane] =
          row_bad ? -1 : static_cast<int32_t>(~static_cast<uint32_t>(best & 0xffffffffull));
    }
    if (lane == 0 && p.dev_status) p.dev_status[r] = row_bad ? DDT_ERR_INPUT : DDT_OK;
  }
  cluster_sync();  // the slices' shared memory stays until the first CTA has read it
}

template <int KM, bool kBF16>
static int launch_dr_t(const DrafterParams& p, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(p.R * p.C));
  cfg.blockDim = dim3(kDrThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = (unsigned)p.C;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, drafter_topk_kernel<KM, kBF16>, p) == cudaSuccess ? DDT_OK : DDT_ERR_CUDA;
}

template <int KM>
static int launch_dr(const DrafterParams& p, cudaStream_t stream) {
  if (p.logits_dtype == DDT_BF16) return launch_dr_t<KM, true>(p, stream);
  return launch_dr_t<KM, false>(p, stream);
}

int launch_drafter_topk(DrafterParams p, cudaStream_t stream) {
  const size_t esz = p.logits_dtype == DDT_BF16 ? 2 : 4;
  p.vec = (reinterpret_cast<uintptr_t>(p.logits) % 16 == 0) && (((size_t)p.V * esz) % 16 == 0);
  // slice starts stay on a 16-byte vector
  auto launch = [&](int C) -> int {
    p.C = C;
    p.chunk = ((p.V + C - 1) / C + 7) / 8 * 8;
    if (p.K <= 8) return launch_dr<8>(p, stream);
    if (p.K <= 16) return launch_dr<16>(p, stream);
    return launch_dr<32>(p, stream);
  };
  // one wave: rows x CTAs per row at most one CTA per SM (each CTA holds an
  // SM's registers), slices of at least 16384 logits, at most 8 CTAs per row
  const int by_rows = std::max(1, sm_count() / std::max(1, p.R));
  const int C = std::max(1, std::min({8, (p.V + 16383) / 16384, by_rows}));
  if (C > 1) {
    if (launch(C) == DDT_OK) return DDT_OK;
    (void)cudaGetLastError();  // clusters of C not schedulable here: one CTA per row
  }
  return launch(1);
}

}  // namespace ddt
