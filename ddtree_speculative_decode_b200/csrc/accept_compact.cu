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
// One launch:
//  * Every (row, vocab-chunk) pair is one CTA that streams its 16-byte
//    vectors once and reduces them to one packed 64-bit key (order-preserving
//    value bits << 32 | ~index): the max key is the largest logit at its
//    lowest index. Partial keys go to the workspace.
//  * The CTA that finishes a request's last chunk (a per-request arrival
//    counter in the workspace; it resets the counter to zero for the next call)
//    folds the partial keys into am[], walks the tree with warp ballots, then
//    copies the accepted rows. path[j] >= j and the path is increasing, so
//    copying rows in increasing j is already read-before-write per byte; the
//    CTA still stages groups of rows in registers behind a barrier so many rows
//    are in flight at once.
#include <mutex>

#include "ddt_kernels.cuh"

namespace ddt {

constexpr int kArgmaxThreads = 256;
constexpr int kArgmaxChunk = 16384;  // vocab entries per CTA

__device__ __forceinline__ unsigned long long pack_key(float v, int idx) {
  return (static_cast<unsigned long long>(float_order_key(v)) << 32) |
         static_cast<unsigned long long>(~static_cast<uint32_t>(idx));
}

__device__ __forceinline__ unsigned long long umax64(unsigned long long a, unsigned long long b) {
  return a > b ? a : b;
}

__device__ __noinline__ void walk_compact_body(const AcceptParams& p, int b);

template <bool kBF16>
__global__ void __launch_bounds__(kArgmaxThreads) accept_kernel(AcceptParams p) {
  pdl_wait();
  pdl_launch_dependents();
  const int row = blockIdx.x / p.chunks;  // b * N + i
  const int chunk = blockIdx.x - row * p.chunks;
  const int b = row / p.N;
  const int i = row - b * p.N;
  const int n = p.n_nodes[b];
  if (i >= n) {
    // an empty tree has no argmax CTAs: one CTA writes its (skipped) outputs
    if (n <= 0 && i == 0 && chunk == 0) walk_compact_body(p, b);
    return;
  }
  const int v0 = chunk * kArgmaxChunk;
  const int v1 = min(p.V, v0 + kArgmaxChunk);
  unsigned long long best = 0ull;
  if (kBF16) {
    const uint16_t* src = static_cast<const uint16_t*>(p.logits) + (size_t)row * p.V;
    // 8 bf16 per 16-byte vector when the row start is 16-byte aligned
    const bool vec = ((reinterpret_cast<uintptr_t>(src + v0) & 15u) == 0);
    if (vec) {
      const int nvec = (v1 - v0) >> 3;
      const uint4* s4 = reinterpret_cast<const uint4*>(src + v0);
      constexpr int U = 8;
      for (int base = 0; base < nvec; base += kArgmaxThreads * U) {
        uint4 r[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int e = base + u * kArgmaxThreads + threadIdx.x;
          r[u] = e < nvec ? __ldcs(s4 + e) : make_uint4(0xff80ff80u, 0xff80ff80u, 0xff80ff80u, 0xff80ff80u);
        }
        // pass 1: the thread's largest value (packed bf16 max, -inf padding)
        __nv_bfloat162 m2 = __halves2bfloat162(__ushort_as_bfloat16(0xff80), __ushort_as_bfloat16(0xff80));
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const uint32_t w[4] = {r[u].x, r[u].y, r[u].z, r[u].w};
#pragma unroll
          for (int t = 0; t < 4; ++t) m2 = __hmax2(m2, *reinterpret_cast<const __nv_bfloat162*>(&w[t]));
        }
        const float mx = fmaxf(__low2float(m2), __high2float(m2));
        // pass 2: its lowest index (values compare as floats, so -0 == +0)
        int first = 0x7fffffff;
#pragma unroll
        for (int u = U - 1; u >= 0; --u) {
          const int e = base + u * kArgmaxThreads + threadIdx.x;
          const uint32_t w[4] = {r[u].x, r[u].y, r[u].z, r[u].w};
#pragma unroll
          for (int t = 3; t >= 0; --t) {
            const int idx = v0 + e * 8 + 2 * t;
            if (e < nvec && __uint_as_float(w[t] & 0xffff0000u) == mx) first = idx + 1;
            if (e < nvec && __uint_as_float(w[t] << 16) == mx) first = idx;
          }
        }
        if (first != 0x7fffffff) best = umax64(best, pack_key(mx, first));
      }
      for (int v = v0 + nvec * 8 + threadIdx.x; v < v1; v += kArgmaxThreads)
        best = umax64(best, pack_key(bf16_bits_to_float(src[v]), v));
    } else {
      for (int v = v0 + threadIdx.x; v < v1; v += kArgmaxThreads)
        best = umax64(best, pack_key(bf16_bits_to_float(src[v]), v));
    }
  } else {
    const float* src = static_cast<const float*>(p.logits) + (size_t)row * p.V;
    const bool vec = ((reinterpret_cast<uintptr_t>(src + v0) & 15u) == 0);
    if (vec) {
      const int nvec = (v1 - v0) >> 2;
      const float4* s4 = reinterpret_cast<const float4*>(src + v0);
      for (int e = threadIdx.x; e < nvec; e += kArgmaxThreads) {
        const float4 r = __ldcs(s4 + e);
        const int idx = v0 + e * 4;
        best = umax64(best, pack_key(r.x, idx));
        best = umax64(best, pack_key(r.y, idx + 1));
        best = umax64(best, pack_key(r.z, idx + 2));
        best = umax64(best, pack_key(r.w, idx + 3));
      }
      for (int v = v0 + nvec * 4 + threadIdx.x; v < v1; v += kArgmaxThreads)
        best = umax64(best, pack_key(src[v], v));
    } else {
      for (int v = v0 + threadIdx.x; v < v1; v += kArgmaxThreads)
        best = umax64(best, pack_key(src[v], v));
    }
  }
  // block reduce: warp shuffles, then one value per warp through shared memory
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) best = umax64(best, __shfl_xor_sync(DDT_FULL_MASK, best, o));
  __shared__ unsigned long long wbest[kArgmaxThreads / 32];
  if ((threadIdx.x & 31) == 0) wbest[threadIdx.x >> 5] = best;
  __syncthreads();
  __shared__ int s_last;
  if (threadIdx.x == 0) {
    unsigned long long m = wbest[0];
#pragma unroll
    for (int w = 1; w < kArgmaxThreads / 32; ++w) m = umax64(m, wbest[w]);
    p.partial[(size_t)row * p.chunks + chunk] = m;
    __threadfence();
    const unsigned prev = atomicAdd(p.counter + b, 1u);
    s_last = (prev == (unsigned)(n * p.chunks - 1));
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  walk_compact_body(p, b);
  if (threadIdx.x == 0) p.counter[b] = 0u;
}

constexpr int kWalkThreads = 256;
constexpr int kMaxN = 1024;
constexpr int kStageRows = 16;  // rows staged per copy round
constexpr int kStageVec = 8;    // 16-byte vectors per thread per round (256 * 8 * 16 B = 32 KB)

__device__ __noinline__ void walk_compact_body(const AcceptParams& p, int b) {
  const int N = p.N;
  const int n = p.n_nodes[b];
  __shared__ int32_t s_am[kMaxN];
  __shared__ int32_t s_path[kMaxN];
  __shared__ int32_t s_par[kMaxN];
  __shared__ int32_t s_tok[kMaxN];
  __shared__ int s_a;
  __shared__ int s_skip;

  if (threadIdx.x == 0) {
    int st = DDT_OK;
    const int L = p.cache_len[b];
    if (n > 0 && (int64_t)L + n > (int64_t)p.cache_cap[b]) st = DDT_ERR_CAPACITY;
    s_skip = (n <= 0 || st != DDT_OK);
    if (p.dev_status) p.dev_status[b] = st;
  }
  // fold partial argmax keys: 4 threads per row, each over a strided subset
  // of the chunks, then a 4-lane shuffle reduce
  for (int i0 = 0; i0 < N; i0 += kWalkThreads / 4) {
    const int i = i0 + (threadIdx.x >> 2);
    const int sub = threadIdx.x & 3;
    unsigned long long m = 0ull;
    if (i < n) {
      const unsigned long long* pk = p.partial + ((size_t)b * N + i) * p.chunks;
      for (int c = sub; c < p.chunks; c += 4) m = umax64(m, __ldcg(pk + c));
    }
    m = umax64(m, __shfl_xor_sync(DDT_FULL_MASK, m, 1));
    m = umax64(m, __shfl_xor_sync(DDT_FULL_MASK, m, 2));
    if (sub == 0 && i < N) {
      const int a = i < n ? static_cast<int>(~static_cast<uint32_t>(m & 0xffffffffull)) : -1;
      s_am[i] = a;
      if (p.am) p.am[(size_t)b * N + i] = a;
    }
  }
  for (int i = threadIdx.x; i < n; i += kWalkThreads) {
    s_par[i] = p.parent[(size_t)b * N + i];
    s_tok[i] = p.node_tok[(size_t)b * N + i];
  }
  __syncthreads();
  const bool skip = s_skip;
  // greedy walk on warp 0
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const int32_t* par = s_par;
    const int32_t* tk = s_tok;
    int a = 0;
    if (!skip) {
      int curn = 0;
      if (lane == 0) s_path[0] = 0;
      for (;;) {
        const int want = s_am[curn];
        int found = -1;
        // children have larger indices than their parent
        for (int base = curn + 1; base < n && found < 0; base += 32) {
          const int c = base + lane;
          const bool hit = c < n && par[c] == curn && tk[c] == want;
          const uint32_t bal = __ballot_sync(DDT_FULL_MASK, hit);
          if (bal) found = base + __ffs(bal) - 1;
        }
        if (found < 0) break;
        ++a;
        if (lane == 0) s_path[a] = found;
        curn = found;
      }
    }
    if (lane == 0) s_a = a;
  }
  __syncthreads();
  const int a = s_a;
  // outputs
  for (int j = threadIdx.x; j < N; j += kWalkThreads) {
    const bool in = !skip && j <= a;
    p.acc_nodes[(size_t)b * N + j] = in ? s_path[j] : -1;
    int t = -1;
    if (in) t = (j < a) ? p.node_tok[(size_t)b * N + s_path[j + 1]] : s_am[s_path[a]];
    p.out_tok[(size_t)b * N + j] = t;
  }
  if (threadIdx.x == 0) {
    p.acc_len[b] = skip ? 0 : a;
    p.bonus[b] = skip ? -1 : s_am[s_path[a]];
  }
  if (skip) return;
  // compaction: rows path[0..a] -> L + 0..a on every layer
  const int L = p.cache_len[b];
  const int rows = a + 1;
  const int64_t base_row = p.cache_off[b] + L;
  const bool v16 = (p.row_bytes % 16 == 0) &&
                   ((reinterpret_cast<uintptr_t>(p.kv) & 15u) == 0) && (p.layer_stride_bytes % 16 == 0);
  for (int layer = 0; layer < p.n_layers; ++layer) {
    unsigned char* lbase = p.kv + layer * p.layer_stride_bytes + base_row * p.row_bytes;
    if (v16) {
      const int vpr = p.row_bytes / 16;  // vectors per row
      for (int r0 = 0; r0 < rows; r0 += kStageRows) {
        const int nr = min(kStageRows, rows - r0);
        const int total = nr * vpr;
        for (int t0 = 0; t0 < total; t0 += kWalkThreads * kStageVec) {
          uint4 buf[kStageVec];
#pragma unroll
          for (int u = 0; u < kStageVec; ++u) {
            const int e = t0 + u * kWalkThreads + threadIdx.x;
            if (e < total) {
              const int rr = e / vpr, cc = e - rr * vpr;
              buf[u] = reinterpret_cast<const uint4*>(lbase + (size_t)s_path[r0 + rr] * p.row_bytes)[cc];
            }
          }
          __syncthreads();
#pragma unroll
          for (int u = 0; u < kStageVec; ++u) {
            const int e = t0 + u * kWalkThreads + threadIdx.x;
            if (e < total) {
              const int rr = e / vpr, cc = e - rr * vpr;
              reinterpret_cast<uint4*>(lbase + (size_t)(r0 + rr) * p.row_bytes)[cc] = buf[u];
            }
          }
          __syncthreads();
        }
      }
    } else {
      const int wpr = p.row_bytes / 4;
      for (int r0 = 0; r0 < rows; r0 += kStageRows) {
        const int nr = min(kStageRows, rows - r0);
        const int total = nr * wpr;
        for (int t0 = 0; t0 < total; t0 += kWalkThreads * kStageVec) {
          uint32_t buf[kStageVec];
#pragma unroll
          for (int u = 0; u < kStageVec; ++u) {
            const int e = t0 + u * kWalkThreads + threadIdx.x;
            if (e < total) {
              const int rr = e / wpr, cc = e - rr * wpr;
              buf[u] = reinterpret_cast<const uint32_t*>(lbase + (size_t)s_path[r0 + rr] * p.row_bytes)[cc];
            }
          }
          __syncthreads();
#pragma unroll
          for (int u = 0; u < kStageVec; ++u) {
            const int e = t0 + u * kWalkThreads + threadIdx.x;
            if (e < total) {
              const int rr = e / wpr, cc = e - rr * wpr;
              reinterpret_cast<uint32_t*>(lbase + (size_t)(r0 + rr) * p.row_bytes)[cc] = buf[u];
            }
          }
          __syncthreads();
        }
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) p.cache_len[b] = L + rows;
}

static size_t counter_bytes(int B) { return ((size_t)B * 4 + 255) / 256 * 256; }

size_t accept_workspace_bytes(int B, int N, int V) {
  const size_t chunks = (size_t)ceil_div(V, kArgmaxChunk);
  return counter_bytes(B) + (size_t)B * N * chunks * sizeof(unsigned long long);
}

int launch_accept_compact(AcceptParams p, void* workspace, cudaStream_t stream) {
  p.chunks = ceil_div(p.V, kArgmaxChunk);
  p.counter = static_cast<unsigned*>(workspace);
  p.partial = reinterpret_cast<unsigned long long*>(static_cast<unsigned char*>(workspace) + counter_bytes(p.B));
  const unsigned grid = (unsigned)p.chunks * (unsigned)(p.B * p.N);
  if (p.logits_dtype == DDT_BF16) return launch_pdl(accept_kernel<true>, grid, kArgmaxThreads, 0, stream, p);
  return launch_pdl(accept_kernel<false>, grid, kArgmaxThreads, 0, stream, p);
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
  static void* ptrs[128] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) {
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
  // the counters must start at zero; the array keeps whatever the last call
  // (on any stream) left there, so clear them on this call's stream first
  if (cudaMemsetAsync(scratch, 0, counter_bytes(p.B), stream) != cudaSuccess) return DDT_ERR_CUDA;
  return launch_accept_compact(p, scratch, stream);
}

}  // namespace ddt
