// Greedy tree accept + latent-KV compaction.
//
// What it computes is fixed in ddt.h (ddt_accept_compact): the target's argmax
// of every verify row, the greedy walk from the root along children whose token
// equals that argmax, and the in-place move of the accepted nodes' latent rows
// into the contiguous cache ("autoregressive_test_driver_kdtree_engine",
// section "The Broader Context": greedy tree-accept kernel, KV cache with
// post-verify compaction; "ddtree_speculative_decode_test_capstone", section
// "What the Test Validated": the bonus token).
//
// Two launches:
//  * accept_argmax_kernel streams the logits once with coalesced 16-byte
//    loads, eight in flight per lane, 32 warps per SM. Work is cut into
//    slices of 2048 entries of one row, handed out to warps in chunks of
//    consecutive slices by atomic counters in the workspace; a warp folds
//    each row's slices of a chunk itself and publishes one
//    packed 64-bit key per row segment with a fire-and-forget atomic max
//    (key = order-preserving value bits << 32 | ~index: the max key is the
//    largest logit at its lowest index). A lane only searches for an index
//    when a batch beats its running maximum, so the common batch costs one
//    packed max per two values. The argmax reads nothing the tree build or
//    the verify attention writes (every row of the logits is reduced, pad
//    rows included), so it starts as soon as the kernel before it lets its
//    dependents launch: its CTAs take SMs the attention leaves idle (its
//    last, ragged wave) and, through the shared counter, most of the work.
//    Each CTA waits for the kernel before it only at its end, so this grid
//    still ends after that kernel.
//  * accept_walk_kernel, one CTA per request (launched programmatically: it
//    stages the tree while the argmax runs), turns the row keys into am[],
//    finds every node's accepted child (the lowest-index child whose token is
//    the node's argmax) with shared-memory atomics, chases the path from the
//    root, writes the outputs, copies the accepted rows and clears the row
//    keys for the next call. path[j] >= j and the path is increasing, so
//    copying rows in increasing j is already read-before-write per byte; rows
//    are still staged in registers behind a barrier so that many are in
//    flight at once.
#include <algorithm>
#include <mutex>

#include "ddt_kernels.cuh"
#include "sm100_ptx.cuh"

namespace ddt {

constexpr int kSliceVec = 8;                      // 16-byte loads per lane per slice
constexpr int kArgmaxThreads = 512;
constexpr int kArgmaxCtasPerSm = 2;
constexpr int kWalkThreads = 512;
constexpr int kMaxN = 1024;
constexpr int kStageVec = 4;                      // 16-byte vectors per thread per copy round
constexpr int kChunkSlices = 4;                   // slices per chunk of the register-fed argmax's work feed

template <bool kBF16>
struct SliceCfg {
  static constexpr int kPer = kBF16 ? 8 : 4;                // values per 16-byte vector
  static constexpr int kElems = 32 * kSliceVec * kPer;      // values per slice
};

__device__ __forceinline__ unsigned long long pack_key(float v, int idx) {
  return (static_cast<unsigned long long>(float_order_key(v)) << 32) |
         static_cast<unsigned long long>(~static_cast<uint32_t>(idx));
}

__device__ __forceinline__ unsigned long long umax64(unsigned long long a, unsigned long long b) {
  return a > b ? a : b;
}

__device__ __forceinline__ unsigned long long warp_max64(unsigned long long k) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) k = umax64(k, __shfl_xor_sync(DDT_FULL_MASK, k, o));
  return k;
}

// Value t (0..kPer-1) of a 16-byte vector.
template <bool kBF16>
__device__ __forceinline__ float vec_val(const uint4& r, int t) {
  const uint32_t w = t < (kBF16 ? 2 : 1) ? r.x : t < (kBF16 ? 4 : 2) ? r.y : t < (kBF16 ? 6 : 3) ? r.z : r.w;
  if (!kBF16) return __uint_as_float(w);
  return __uint_as_float((t & 1) ? (w & 0xffff0000u) : (w << 16));
}

// Work feed: chunks of `chunk` consecutive slices handed out by counters in
// the workspace header (kCounters of them, 32 bytes apart; a warp draws from
// counter gw % kCounters, which serves chunks ctr, ctr + kCounters, ...), so
// warps that start early -- beside the kernel before this one -- take more of
// the work. Lane 0 keeps the next draw in flight while the current chunk is
// read. (A static first chunk per warp, or several draws in flight per warp,
// measured slower steps.)
constexpr int kCounters = 7;
struct ChunkFeed {
  unsigned* work;
  long long slices, chunk, nchunks;
  int ctr;             // this warp's counter
  unsigned pre;        // lane 0: the next counter value (in flight)
  long long cs, ce;    // warp-uniform: the current chunk's slices [cs, ce)
  __device__ void start(long long gw, int lane) {
    ctr = (int)(gw % kCounters);
    cs = ce = 0;
    pre = lane == 0 ? atomicAdd(work + 8 * ctr, 1u) : 0u;
  }
  // the warp's next slice, or -1 once its counter is past the last chunk
  // (every later draw of that counter is larger)
  __device__ long long next(int lane) {
    if (cs >= ce) {
      const long long c = (long long)__shfl_sync(DDT_FULL_MASK, pre, 0) * kCounters + ctr;
      if (c >= nchunks) return -1;
      if (lane == 0) pre = atomicAdd(work + 8 * ctr, 1u);
      cs = c * chunk;
      ce = cs + chunk < slices ? cs + chunk : slices;
    }
    return cs++;
  }
};

template <bool kBF16>
__global__ void __launch_bounds__(kArgmaxThreads) accept_argmax_kernel(AcceptParams p) {
  using C = SliceCfg<kBF16>;
  // no wait for the kernel before: see the file comment (it comes at the end)
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int spr = (p.V + C::kElems - 1) / C::kElems;  // slices per row
  const long long slices = (long long)p.B * p.N * spr;
  const long long gw = ((long long)blockIdx.x * kArgmaxThreads + threadIdx.x) >> 5;
  ChunkFeed feed{p.work, slices, kChunkSlices, (slices + kChunkSlices - 1) / kChunkSlices};
  feed.start(gw, lane);
  const size_t esz = kBF16 ? 2 : 4;
  int cur_row = -1;
  float best_v = -INFINITY;   // this lane's running max of cur_row and its lowest index
  int best_i = -1;
  auto flush = [&]() {
    const unsigned long long k = warp_max64(best_i < 0 ? 0ull : pack_key(best_v, best_i));
    if (lane == 0 && k != 0ull) atomicMax(p.rowkey + cur_row, k);  // result unused: no wait
  };
  for (long long sl = feed.next(lane); sl >= 0; sl = feed.next(lane)) {
    const int r = (int)(sl / spr), c = (int)(sl - (long long)r * spr);
    if (r != cur_row) {
      if (cur_row >= 0) flush();
      cur_row = r;
      best_v = -INFINITY;
      best_i = -1;
    }
    const int v0 = c * C::kElems;
    const int cnt = min(C::kElems, p.V - v0);
    const unsigned char* row = static_cast<const unsigned char*>(p.logits) + ((size_t)r * p.V + v0) * esz;
    if (p.tma) {  // 16-byte aligned rows: cnt is a multiple of kPer
      const int nvec = cnt / C::kPer;
      uint4 v[kSliceVec];
#pragma unroll
      for (int k = 0; k < kSliceVec; ++k) {
        const int e = lane + 32 * k;
        v[k] = e < nvec ? __ldcs(reinterpret_cast<const uint4*>(row) + e)
                        : (kBF16 ? make_uint4(0xff80ff80u, 0xff80ff80u, 0xff80ff80u, 0xff80ff80u)
                                 : make_uint4(0xff800000u, 0xff800000u, 0xff800000u, 0xff800000u));
      }
      // tree-shaped maximum (short dependency chains)
      float m;
      if (kBF16) {
        auto h = [](uint32_t w) { return *reinterpret_cast<const __nv_bfloat162*>(&w); };
        __nv_bfloat162 mk[kSliceVec];
#pragma unroll
        for (int k = 0; k < kSliceVec; ++k)
          mk[k] = __hmax2(__hmax2(h(v[k].x), h(v[k].y)), __hmax2(h(v[k].z), h(v[k].w)));
#pragma unroll
        for (int w = kSliceVec / 2; w > 0; w >>= 1)
#pragma unroll
          for (int k = 0; k < w; ++k) mk[k] = __hmax2(mk[k], mk[k + w]);
        m = fmaxf(__low2float(mk[0]), __high2float(mk[0]));
      } else {
        float mk[kSliceVec];
#pragma unroll
        for (int k = 0; k < kSliceVec; ++k)
          mk[k] = fmaxf(fmaxf(__uint_as_float(v[k].x), __uint_as_float(v[k].y)),
                        fmaxf(__uint_as_float(v[k].z), __uint_as_float(v[k].w)));
#pragma unroll
        for (int w = kSliceVec / 2; w > 0; w >>= 1)
#pragma unroll
          for (int k = 0; k < w; ++k) mk[k] = fmaxf(mk[k], mk[k + w]);
        m = mk[0];
      }
      const bool has_real = lane < nvec;
      if (has_real && (m > best_v || best_i < 0)) {
        // lowest real index holding m (values compare as floats: -0 == +0)
        int first = -1;
#pragma unroll
        for (int k = kSliceVec - 1; k >= 0; --k) {
          const int e = lane + 32 * k;
#pragma unroll
          for (int t = C::kPer - 1; t >= 0; --t)
            if (e < nvec && vec_val<kBF16>(v[k], t) == m) first = v0 + e * C::kPer + t;
        }
        best_v = m;
        best_i = first;
      }
    } else {
      for (int t = lane; t < cnt; t += 32) {
        const float x = kBF16 ? bf16_bits_to_float(reinterpret_cast<const uint16_t*>(row)[t])
                              : reinterpret_cast<const float*>(row)[t];
        if (x > best_v || best_i < 0) { best_v = x; best_i = v0 + t; }
      }
    }
  }
  if (cur_row >= 0) flush();
  pdl_wait();  // this grid ends after the kernel before it (the walk relies on that)
}

// The same argmax for 16-byte aligned rows, fed by 1-D bulk copies: each
// warp streams the slices of its chunks through a ring of kBulkBufs
// shared-memory buffers (one mbarrier each), so every SM keeps 192 KB of
// logits in flight -- more than registers can hold -- and a launch of few
// rows finishes in one round trip to HBM.
constexpr int kBulkWarps = kArgmaxThreads / 32;
constexpr int kBulkBufs = 3;
constexpr int kSliceBytes = 32 * kSliceVec * 16;
constexpr int kBulkSmem = kBulkWarps * kBulkBufs * (kSliceBytes + 8);

template <bool kBF16>
__global__ void __launch_bounds__(kArgmaxThreads, 1) accept_argmax_bulk_kernel(AcceptParams p) {
  using C = SliceCfg<kBF16>;
  extern __shared__ __align__(128) unsigned char smem[];
  // no wait for the kernel before: see the file comment (it comes at the end)
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // a status word already holding an error (an earlier wait gave up): nothing to do
  if (*reinterpret_cast<const volatile int*>(p.status_word) != 0) {
    pdl_wait();
    return;
  }
  const int spr = (p.V + C::kElems - 1) / C::kElems;  // slices per row
  const long long slices = (long long)p.B * p.N * spr;
  const long long gw = (long long)blockIdx.x * kBulkWarps + warp;
  // single slices: few rows give each warp only a couple
  ChunkFeed feed{p.work, slices, 1, slices};
  const size_t esz = kBF16 ? 2 : 4;
  unsigned char* wbuf = smem + warp * kBulkBufs * kSliceBytes;
  const uint32_t bar0 = sm100::smem_u32(smem + kBulkWarps * kBulkBufs * kSliceBytes + warp * kBulkBufs * 8);
  if (lane == 0) {
    for (int k = 0; k < kBulkBufs; ++k) sm100::mbar_init(bar0 + 8u * k, 1);
    sm100::fence_mbar_init_cluster();
  }
  __syncwarp();
  feed.start(gw, lane);
  auto issue = [&](long long sl, int k) {  // lane 0
    const int r = (int)(sl / spr), c = (int)(sl - (long long)r * spr);
    const int v0 = c * C::kElems;
    const uint32_t bytes = (uint32_t)(min(C::kElems, p.V - v0) * esz);
    const unsigned char* src = static_cast<const unsigned char*>(p.logits) + ((size_t)r * p.V + v0) * esz;
    sm100::mbar_arrive_expect_tx(bar0 + 8u * k, bytes);
    sm100::bulk_load_1d(sm100::smem_u32(wbuf + k * kSliceBytes), src, bytes, bar0 + 8u * k);
  };
  long long qs[kBulkBufs];
  uint32_t phases = 0;
  long long next = feed.next(lane);
  int issued = 0;
  for (int k = 0; k < kBulkBufs && next >= 0; ++k) {
    if (lane == 0) issue(next, k);
    qs[k] = next;
    next = feed.next(lane);
    ++issued;
  }
  int cur_row = -1;
  float best_v = -INFINITY;
  int best_i = -1;
  auto flush = [&]() {
    const unsigned long long k = warp_max64(best_i < 0 ? 0ull : pack_key(best_v, best_i));
    if (lane == 0 && k != 0ull) atomicMax(p.rowkey + cur_row, k);
  };
  for (int done = 0; done < issued; ++done) {
    const int k = done % kBulkBufs;
    const long long sl = qs[k];
    if (!sm100::mbar_wait(bar0 + 8u * k, (phases >> k) & 1u, p.abort, p.wait_ns)) {
      // gave up: the copies still in flight land in this CTA's shared memory,
      // so wait (bounded) for them before leaving
      for (int j = done; j < issued; ++j) {
        const int kj = j % kBulkBufs;
        (void)sm100::mbar_wait_own(bar0 + 8u * kj, (phases >> kj) & 1u, p.abort, p.wait_ns);
        phases ^= 1u << kj;
      }
      pdl_wait();
      return;
    }
    phases ^= 1u << k;
    const int r = (int)(sl / spr), c = (int)(sl - (long long)r * spr);
    if (r != cur_row) {
      if (cur_row >= 0) flush();
      cur_row = r;
      best_v = -INFINITY;
      best_i = -1;
    }
    const int v0 = c * C::kElems;
    const int nvec = min(C::kElems, p.V - v0) / C::kPer;
    const uint4* src = reinterpret_cast<const uint4*>(wbuf + k * kSliceBytes);
    uint4 v[kSliceVec];
#pragma unroll
    for (int kk = 0; kk < kSliceVec; ++kk) {
      const int e = lane + 32 * kk;
      v[kk] = e < nvec ? src[e]
                       : (kBF16 ? make_uint4(0xff80ff80u, 0xff80ff80u, 0xff80ff80u, 0xff80ff80u)
                                : make_uint4(0xff800000u, 0xff800000u, 0xff800000u, 0xff800000u));
    }
    __syncwarp();  // every lane has read the buffer: it may be refilled
    if (next >= 0) {
      if (lane == 0) issue(next, k);
      qs[k] = next;
      next = feed.next(lane);
      ++issued;
    }
    float m;
    if (kBF16) {
      auto h = [](uint32_t w) { return *reinterpret_cast<const __nv_bfloat162*>(&w); };
      __nv_bfloat162 mk[kSliceVec];
#pragma unroll
      for (int kk = 0; kk < kSliceVec; ++kk)
        mk[kk] = __hmax2(__hmax2(h(v[kk].x), h(v[kk].y)), __hmax2(h(v[kk].z), h(v[kk].w)));
#pragma unroll
      for (int w = kSliceVec / 2; w > 0; w >>= 1)
#pragma unroll
        for (int kk = 0; kk < w; ++kk) mk[kk] = __hmax2(mk[kk], mk[kk + w]);
      m = fmaxf(__low2float(mk[0]), __high2float(mk[0]));
    } else {
      float mk[kSliceVec];
#pragma unroll
      for (int kk = 0; kk < kSliceVec; ++kk)
        mk[kk] = fmaxf(fmaxf(__uint_as_float(v[kk].x), __uint_as_float(v[kk].y)),
                       fmaxf(__uint_as_float(v[kk].z), __uint_as_float(v[kk].w)));
#pragma unroll
      for (int w = kSliceVec / 2; w > 0; w >>= 1)
#pragma unroll
        for (int kk = 0; kk < w; ++kk) mk[kk] = fmaxf(mk[kk], mk[kk + w]);
      m = mk[0];
    }
    if (lane < nvec && (m > best_v || best_i < 0)) {
      int first = -1;  // lowest real index holding m (values compare as floats: -0 == +0)
#pragma unroll
      for (int kk = kSliceVec - 1; kk >= 0; --kk) {
        const int e = lane + 32 * kk;
#pragma unroll
        for (int t = C::kPer - 1; t >= 0; --t)
          if (e < nvec && vec_val<kBF16>(v[kk], t) == m) first = v0 + e * C::kPer + t;
      }
      best_v = m;
      best_i = first;
    }
  }
  if (cur_row >= 0) flush();
  pdl_wait();  // this grid ends after the kernel before it (the walk relies on that)
}

// Request epilogue: one CTA per request.
__global__ void __launch_bounds__(kWalkThreads) accept_walk_kernel(AcceptParams p) {
  __shared__ int32_t s_am[kMaxN];
  __shared__ int32_t s_child[kMaxN];
  __shared__ int32_t s_path[kMaxN];
  __shared__ int32_t s_par[kMaxN];
  __shared__ int32_t s_tok[kMaxN];
  __shared__ int s_misc[3];
  const int b = blockIdx.x, tid = threadIdx.x;
  const int N = p.N;
  // the argmax before this kernel starts without waiting for the tree build
  // and waits for the kernels before it only at its end, so the tree, the
  // cache bookkeeping and the row keys are all read after this wait, in one
  // round of independent loads
  pdl_wait();
  // no early trigger of the next kernel: this one writes the pool and
  // cache_len, which a following verify attention reads before it waits
  constexpr int kPer = kMaxN / kWalkThreads;
  const int n_raw = p.n_nodes[b];
  int L0 = 0, cap0 = 0, sw = 0;  // thread 0's copies
  int64_t off0 = 0;
  if (tid == 0) {
    L0 = p.cache_len[b];
    off0 = p.cache_off[b];
    cap0 = p.cache_cap[b];
    if (p.status_word != nullptr) sw = *reinterpret_cast<const volatile int*>(p.status_word);
  }
  int32_t r_par[kPer], r_tok[kPer];
  unsigned long long r_key[kPer];
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int i = tid + u * kWalkThreads;
    if (i < N) {
      r_par[u] = p.parent[(size_t)b * N + i];
      r_tok[u] = p.node_tok[(size_t)b * N + i];
      r_key[u] = p.rowkey[(size_t)b * N + i];
    }
  }
  // a node count outside [0, N] is bad input: the request is skipped, and
  // only [0, N) is ever indexed
  const int n = min(max(n_raw, 0), N);
  if (tid == 0) {
    int st = DDT_OK;
    // the rows the compaction may touch on every layer, l * stride + off +
    // [L, L + n), must lie in the pool
    const int64_t last = (int64_t)(p.n_layers - 1) * (p.layer_stride_bytes / p.row_bytes) + off0 + L0 + n;
    if (n_raw > N) st = DDT_ERR_INPUT;
    else if (n > 0 && (off0 < 0 || L0 < 0 || last > p.kv_rows)) st = DDT_ERR_BOUNDS;
    else if (n > 0 && (int64_t)L0 + n > (int64_t)cap0) st = DDT_ERR_CAPACITY;
    bool skip = n <= 0 || st != DDT_OK;
    // the kernel that produced the row keys gave up a wait: they are not
    // complete, so nothing is accepted (the keys are still cleared)
    if (sw != 0) {
      skip = true;
      st = DDT_ERR_TIMEOUT;
    }
    s_misc[0] = skip;
    if (p.dev_status) p.dev_status[b] = st;
    // the argmax's work counters back to zero for the next call (its grid has ended)
    if (b == 0 && p.work != nullptr)
      for (int k = 0; k < kCounters; ++k) p.work[8 * k] = 0u;
  }
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int i = tid + u * kWalkThreads;
    if (i < N) {
      int a = -1;
      p.rowkey[(size_t)b * N + i] = 0ull;  // zero for the next call (pad rows have keys too)
      if (i < n) {
        a = static_cast<int>(~static_cast<uint32_t>(r_key[u] & 0xffffffffull));
        s_am[i] = a;
        s_par[i] = r_par[u];
        s_tok[i] = r_tok[u];
        s_child[i] = 0x7fffffff;
      }
      if (p.am) p.am[(size_t)b * N + i] = a;
    }
  }
  __syncthreads();
  const bool skip = s_misc[0] != 0;
  // accepted child of every node: the lowest-index child whose token is the
  // node's argmax (children have larger indices than their parent)
  if (!skip)
    for (int j = 1 + tid; j < n; j += kWalkThreads) {
      const int pp = s_par[j];
      if (pp >= 0 && pp < j && s_tok[j] == s_am[pp]) atomicMin(&s_child[pp], j);
    }
  __syncthreads();
  if (tid == 0) {
    int a = 0, cur = 0;
    s_path[0] = 0;
    if (!skip) {
      for (;;) {
        const int c = s_child[cur];
        if (c >= n) break;  // none
        s_path[++a] = c;
        cur = c;
      }
    }
    s_misc[1] = a;
    s_misc[2] = skip ? -1 : s_am[cur];
  }
  __syncthreads();
  const int a = s_misc[1];
  const int bonus = s_misc[2];
  for (int j = tid; j < N; j += kWalkThreads) {
    const bool in = !skip && j <= a;
    p.acc_nodes[(size_t)b * N + j] = in ? s_path[j] : -1;
    int t = -1;
    if (in) t = (j < a) ? s_tok[s_path[j + 1]] : bonus;
    p.out_tok[(size_t)b * N + j] = t;
  }
  if (tid == 0) {
    p.acc_len[b] = skip ? 0 : a;
    p.bonus[b] = bonus;
  }
  if (skip) return;
  // compaction: rows path[0..a] -> L + 0..a on every layer (several layers:
  // compact_layers_kernel does it, spread over CTAs, after this kernel)
  const int L = p.cache_len[b];
  const int rows = a + 1;
  if (p.layers_apart) {
    __syncthreads();
    if (tid == 0) p.cache_len[b] = L + rows;
    return;
  }
  const int64_t base_row = p.cache_off[b] + L;
  const bool v16 = (p.row_bytes % 16 == 0) && ((reinterpret_cast<uintptr_t>(p.kv) & 15u) == 0) &&
                   (p.layer_stride_bytes % 16 == 0);
  const int vb = v16 ? 16 : 4;         // bytes per vector
  const int vpr = p.row_bytes / vb;    // vectors per row
  const int per_layer = rows * vpr;
  const long long total = (long long)per_layer * p.n_layers;
  for (long long t0 = 0; t0 < total; t0 += (long long)kWalkThreads * kStageVec) {
    uint4 buf[kStageVec];
#pragma unroll
    for (int u = 0; u < kStageVec; ++u) {
      const long long e = t0 + u * kWalkThreads + tid;
      if (e < total) {
        const int layer = (int)(e / per_layer);
        const int rem = (int)(e - (long long)layer * per_layer);
        const int rr = rem / vpr, cc = rem - rr * vpr;
        const unsigned char* src =
            p.kv + layer * p.layer_stride_bytes + (base_row + s_path[rr]) * p.row_bytes + (size_t)cc * vb;
        if (v16) buf[u] = *reinterpret_cast<const uint4*>(src);
        else buf[u].x = *reinterpret_cast<const uint32_t*>(src);
      }
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < kStageVec; ++u) {
      const long long e = t0 + u * kWalkThreads + tid;
      if (e < total) {
        const int layer = (int)(e / per_layer);
        const int rem = (int)(e - (long long)layer * per_layer);
        const int rr = rem / vpr, cc = rem - rr * vpr;
        unsigned char* dst = p.kv + layer * p.layer_stride_bytes + (base_row + rr) * p.row_bytes + (size_t)cc * vb;
        if (v16) *reinterpret_cast<uint4*>(dst) = buf[u];
        else *reinterpret_cast<uint32_t*>(dst) = buf[u].x;
      }
    }
    __syncthreads();
  }
  if (tid == 0) p.cache_len[b] = L + rows;
}

// Multi-layer compaction after the walk: CTA (b, g) moves request b's
// accepted rows on layers [g * per, (g + 1) * per). The walk has written the
// path (acc_nodes, -1 in slot 0 for a skipped request), acc_len and the new
// cache_len, so the committed rows start at cache_len - (acc_len + 1). Rows
// move in rounds of increasing destination index, each round read completely
// before it is written: a path is increasing with path[j] >= j, so no round
// writes a row a later round still reads.
constexpr int kCopyThreads = 256;

__global__ void __launch_bounds__(kCopyThreads) compact_layers_kernel(AcceptParams p, int groups, int per) {
  __shared__ int32_t s_path[kMaxN];
  pdl_wait();  // (no early trigger of the next kernel: this one writes the pool)
  const int b = blockIdx.x / groups, g = blockIdx.x - b * groups;
  const int tid = threadIdx.x;
  const int N = p.N;
  if (p.acc_nodes[(size_t)b * N] != 0) return;  // skipped request: nothing moves
  const int rows = p.acc_len[b] + 1;
  for (int j = tid; j < rows; j += kCopyThreads) s_path[j] = p.acc_nodes[(size_t)b * N + j];
  __syncthreads();
  const int64_t base_row = p.cache_off[b] + (p.cache_len[b] - rows);
  const int l0 = g * per, l1 = min(p.n_layers, l0 + per);
  const bool v16 = (p.row_bytes % 16 == 0) && ((reinterpret_cast<uintptr_t>(p.kv) & 15u) == 0) &&
                   (p.layer_stride_bytes % 16 == 0);
  const int vb = v16 ? 16 : 4;
  const int vpr = p.row_bytes / vb;
  const long long per_layer = (long long)rows * vpr;
  const long long total = per_layer * (l1 - l0);
  for (long long t0 = 0; t0 < total; t0 += (long long)kCopyThreads * kStageVec) {
    uint4 buf[kStageVec];
#pragma unroll
    for (int u = 0; u < kStageVec; ++u) {
      const long long e = t0 + u * kCopyThreads + tid;
      if (e < total) {
        const int layer = l0 + (int)(e / per_layer);
        const long long rem = e % per_layer;
        const int rr = (int)(rem / vpr), cc = (int)(rem - (long long)rr * vpr);
        const unsigned char* src =
            p.kv + layer * p.layer_stride_bytes + (base_row + s_path[rr]) * p.row_bytes + (size_t)cc * vb;
        if (v16) buf[u] = __ldcs(reinterpret_cast<const uint4*>(src));
        else buf[u].x = *reinterpret_cast<const uint32_t*>(src);
      }
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < kStageVec; ++u) {
      const long long e = t0 + u * kCopyThreads + tid;
      if (e < total) {
        const int layer = l0 + (int)(e / per_layer);
        const long long rem = e % per_layer;
        const int rr = (int)(rem / vpr), cc = (int)(rem - (long long)rr * vpr);
        unsigned char* dst = p.kv + layer * p.layer_stride_bytes + (base_row + rr) * p.row_bytes + (size_t)cc * vb;
        if (v16) *reinterpret_cast<uint4*>(dst) = buf[u];
        else *reinterpret_cast<uint32_t*>(dst) = buf[u].x;
      }
    }
    __syncthreads();
  }
}

// Launch the walk, then (several layers) the spread-out compaction.
static int launch_walk_and_copy(AcceptParams p, cudaStream_t stream) {
  p.layers_apart = p.n_layers > 1 ? 1 : 0;
  const int st = launch_pdl(accept_walk_kernel, (unsigned)p.B, kWalkThreads, 0, stream, p);
  if (st != DDT_OK || !p.layers_apart) return st;
  // about two CTAs per SM over all requests, whole layers per CTA
  const int groups = std::max(1, std::min(p.n_layers, ceil_div(2 * sm_count(), p.B)));
  const int per = ceil_div(p.n_layers, groups);
  const int used = ceil_div(p.n_layers, per);
  return launch_pdl(compact_layers_kernel, (unsigned)(p.B * used), kCopyThreads, 0, stream, p, used, per);
}

static size_t round256(size_t x) { return (x + 255) / 256 * 256; }
static size_t header_bytes() { return 256; }
constexpr size_t kWorkCounterOffset = 32;  // the argmax's work counters: header bytes 32, 64, ..., 224
static size_t zeroed_bytes(int B, int N) { return header_bytes() + round256((size_t)B * N * 8); }

size_t accept_workspace_bytes(int B, int N, int V) {
  (void)V;
  return zeroed_bytes(B, N);
}


// The bulk-copy argmax's shared-memory opt-in, set once per device.
static bool bulk_argmax_ready(bool bf16) {
  static std::mutex mu;
  static int done[kMaxDevices][2] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lock(mu);
  int& d = done[dev][bf16 ? 1 : 0];
  if (d == 0) {
    const cudaError_t e =
        bf16 ? cudaFuncSetAttribute(accept_argmax_bulk_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    kBulkSmem)
             : cudaFuncSetAttribute(accept_argmax_bulk_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    kBulkSmem);
    d = e == cudaSuccess ? 1 : -1;
    if (e != cudaSuccess) (void)cudaGetLastError();
  }
  return d == 1;
}

int launch_accept_compact(AcceptParams p, void* workspace, cudaStream_t stream) {
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  // the first 256 bytes: status word (a bounded wait of the argmax gave up)
  // at byte 0, the argmax's work counters at bytes 32, 64, ..., 224
  p.abort = reinterpret_cast<int*>(ws);
  p.status_word = reinterpret_cast<const int*>(ws);
  p.work = reinterpret_cast<unsigned*>(ws + kWorkCounterOffset);
  p.wait_ns = wait_limit_ns();
  p.rowkey = reinterpret_cast<unsigned long long*>(ws + header_bytes());
  const size_t esz = p.logits_dtype == DDT_BF16 ? 2 : 4;
  p.tma = (reinterpret_cast<uintptr_t>(p.logits) % 16 == 0) && (((size_t)p.V * esz) % 16 == 0);
  const int elems = p.logits_dtype == DDT_BF16 ? SliceCfg<true>::kElems : SliceCfg<false>::kElems;
  const long long slices = (long long)p.B * p.N * ceil_div(p.V, elems);
  const bool bf = p.logits_dtype == DDT_BF16;
  // the register-fed kernel keeps 128 KB per SM in flight: enough when the
  // logits take several rounds of it; a launch of few rows (fewer slices
  // than two of its rounds) finishes sooner with the bulk-copy ring, which
  // keeps 192 KB per SM in flight (measured: 64 rows x 163840, 14.6 against
  // 15.4 us per accept; 512 rows, 48 against 43 us)
  const long long reg_warps = (long long)sm_count() * kArgmaxCtasPerSm * (kArgmaxThreads / 32);
  int st;
  if (p.tma && slices <= 2 * reg_warps && bulk_argmax_ready(bf)) {
    // at most one CTA of 16 warps per SM; warps take chunks of slices
    const unsigned grid = (unsigned)std::max(1LL, std::min<long long>(sm_count(), ceil_div((int)std::min<long long>(
                                                                                               slices, 1LL << 30),
                                                                                           kBulkWarps)));
    st = bf ? launch_pdl(accept_argmax_bulk_kernel<true>, grid, kArgmaxThreads, (size_t)kBulkSmem, stream, p)
            : launch_pdl(accept_argmax_bulk_kernel<false>, grid, kArgmaxThreads, (size_t)kBulkSmem, stream, p);
  } else {
    const long long warps = std::max(1LL, std::min<long long>(slices, (long long)sm_count() * kArgmaxCtasPerSm *
                                                                          (kArgmaxThreads / 32)));
    const unsigned grid = (unsigned)((warps + kArgmaxThreads / 32 - 1) / (kArgmaxThreads / 32));
    st = bf ? launch_pdl(accept_argmax_kernel<true>, grid, kArgmaxThreads, 0, stream, p)
            : launch_pdl(accept_argmax_kernel<false>, grid, kArgmaxThreads, 0, stream, p);
  }
  if (st != DDT_OK) return st;
  return launch_walk_and_copy(p, stream);
}

// The walk and compaction alone, on row keys another kernel (the LM-head
// argmax) left in the workspace; a non-zero status word there means that
// kernel gave up.
int launch_accept_walk(AcceptParams p, void* workspace, cudaStream_t stream) {
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  p.rowkey = reinterpret_cast<unsigned long long*>(ws + header_bytes());
  p.status_word = reinterpret_cast<const int*>(ws);
  p.work = reinterpret_cast<unsigned*>(ws + kWorkCounterOffset);
  return launch_walk_and_copy(p, stream);
}

// ---------------------------------------------------------------------------
// Allocation-free variant: the same kernel, with its scratch (per-request
// arrival counters + partial argmax keys) in a fixed device array that is part
// of the loaded library instead of a caller-provided workspace.
// ---------------------------------------------------------------------------

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;  // 4 MiB on every device that loads the library
static __device__ __align__(256) unsigned char g_accept_scratch[kNoAllocScratchBytes];

size_t accept_noalloc_scratch_bytes() { return kNoAllocScratchBytes; }

// Device address of g_accept_scratch, looked up once per device (with that
// device current). Host code must not hand the symbol itself to a kernel: on
// the host it names a stand-in, not device memory.
static void* noalloc_scratch_ptr(int* status) {
  static std::mutex mu;
  static void* ptrs[kMaxDevices] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    *status = DDT_ERR_CUDA;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (ptrs[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_accept_scratch) != cudaSuccess || ptr == nullptr) {
      *status = DDT_ERR_CUDA;
      return nullptr;
    }
    ptrs[dev] = ptr;
  }
  *status = DDT_OK;
  return ptrs[dev];
}

int launch_accept_compact_noalloc(AcceptParams p, cudaStream_t stream) {
  if (accept_workspace_bytes(p.B, p.N, p.V) > kNoAllocScratchBytes) return DDT_ERR_UNSUPPORTED;
  int st = DDT_OK;
  void* scratch = noalloc_scratch_ptr(&st);
  if (st != DDT_OK) return st;
  // the status word and row keys must start at zero; the array keeps
  // whatever the last call (on any stream) left there, so clear them on this
  // call's stream first
  if (cudaMemsetAsync(scratch, 0, zeroed_bytes(p.B, p.N), stream) != cudaSuccess) return DDT_ERR_CUDA;
  return launch_accept_compact(p, scratch, stream);
}

}  // namespace ddt
