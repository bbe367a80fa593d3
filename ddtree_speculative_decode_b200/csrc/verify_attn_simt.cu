// CUDA-core tree-verify attention (float32 accumulation, any d_l / d_r with
// d_qk <= 1024). Serves float32 inputs (the tiny fp32 workload) and every
// shape the tensor-core kernel does not cover.
//
// What it computes is fixed in ddt.h (ddt_verify_attn): for each tree node's
// head, softmax over the committed cache rows plus the tree rows its
// visibility mask selects, of scale * q . kv_row, applied to the rows' first
// d_l entries ("autoregressive_test_driver_kdtree_engine", section "The
// Broader Context": tree-verify MLA-absorb attention with visibility masking).
//
// One warp owns one (request, node, head) row: lanes split the d_qk dims of
// each key row (coalesced row reads), a butterfly shuffle finishes the dot
// product, and an online softmax in the base-2 domain keeps one running max,
// one running sum and d_l / 32 output accumulators per lane.
#include "ddt_kernels.cuh"

namespace ddt {

constexpr int kSimtWarps = 4;
constexpr int kMaxPerLane = 32;  // d_qk <= 1024

template <typename T>
__device__ __forceinline__ float ld_elem(const T* p, int i);
template <>
__device__ __forceinline__ float ld_elem<float>(const float* p, int i) { return p[i]; }
template <>
__device__ __forceinline__ float ld_elem<uint16_t>(const uint16_t* p, int i) { return bf16_bits_to_float(p[i]); }

template <typename Tin, int PL>
__global__ void __launch_bounds__(32 * kSimtWarps) attn_simt_kernel(AttnParams p) {
  pdl_wait();
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * kSimtWarps + warp;  // ((b * N) + i) * H + h
  const long long total = (long long)p.B * p.N * p.H;
  if (row >= total) return;
  const int i = (int)((row / p.H) % p.N);
  const int b = (int)(row / ((long long)p.H * p.N));
  const int d_qk = p.d_l + p.d_r;
  const int n_raw = p.n_nodes[b];
  // a request whose rows do not lie in the pool (or whose node count is
  // outside [0, N]) reads nothing: all its rows are written as pad rows
  const bool oob = n_raw < 0 || n_raw > p.N || p.cache_off[b] < 0 || p.cache_len[b] < 0 ||
                   p.cache_off[b] + p.cache_len[b] + n_raw > p.kv_rows;
  const int n = oob ? 0 : n_raw;
  if (p.dev_status && i == 0 && (row % p.H) == 0 && lane == 0) p.dev_status[b] = oob ? DDT_ERR_BOUNDS : DDT_OK;

  float* lse_out = p.lse ? p.lse + row : nullptr;
  if (i >= n) {
    for (int c = lane; c < p.d_l; c += 32) {
      if (p.out_dtype == DDT_F32)
        static_cast<float*>(p.out)[row * p.d_l + c] = 0.0f;
      else
        static_cast<__nv_bfloat16*>(p.out)[row * p.d_l + c] = __float2bfloat16_rn(0.0f);
    }
    if (lse_out && lane == 0) *lse_out = -INFINITY;
    return;
  }
  const Tin* qrow = static_cast<const Tin*>(p.q) + row * d_qk;
  float qv[PL];
#pragma unroll
  for (int u = 0; u < PL; ++u) {
    const int c = lane + 32 * u;
    qv[u] = c < d_qk ? ld_elem(qrow, c) : 0.0f;
  }
  const float kLog2e = 1.4426950408889634f;
  const float sl2 = p.scale * kLog2e;
  float m = -INFINITY, l = 0.0f;
  float acc[PL];
#pragma unroll
  for (int u = 0; u < PL; ++u) acc[u] = 0.0f;

  const int L = p.cache_len[b];
  const Tin* kvb = static_cast<const Tin*>(p.kv) + p.cache_off[b] * (long long)d_qk;
  const uint32_t* mrow = p.mask + ((size_t)b * p.N + i) * p.W;
  const int nkeys = L + n;
  for (int j = 0; j < nkeys; ++j) {
    if (j >= L) {
      const int t = j - L;
      if (!((mrow[t >> 5] >> (t & 31)) & 1u)) continue;
    }
    const Tin* krow = kvb + (long long)j * d_qk;
    float kvv[PL];
    float part = 0.0f;
#pragma unroll
    for (int u = 0; u < PL; ++u) {
      const int c = lane + 32 * u;
      kvv[u] = c < d_qk ? ld_elem(krow, c) : 0.0f;
      part = fmaf(qv[u], kvv[u], part);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(DDT_FULL_MASK, part, o);
    const float s2 = part * sl2;
    const float mn = fmaxf(m, s2);
    const float alpha = exp2f(m - mn);  // m = -inf on the first key gives 0
    const float pj = exp2f(s2 - mn);
    l = l * alpha + pj;
#pragma unroll
    for (int u = 0; u < PL; ++u) {
      const int c = lane + 32 * u;
      const float v = c < p.d_l ? kvv[u] : 0.0f;
      acc[u] = fmaf(pj, v, acc[u] * alpha);
    }
    m = mn;
  }
  const float inv = l > 0.0f ? 1.0f / l : 0.0f;
#pragma unroll
  for (int u = 0; u < PL; ++u) {
    const int c = lane + 32 * u;
    if (c < p.d_l) {
      const float o = acc[u] * inv;
      if (p.out_dtype == DDT_F32)
        static_cast<float*>(p.out)[row * p.d_l + c] = o;
      else
        static_cast<__nv_bfloat16*>(p.out)[row * p.d_l + c] = __float2bfloat16_rn(o);
    }
  }
  if (lse_out && lane == 0) *lse_out = l > 0.0f ? (m + log2f(l)) * 0.6931471805599453f : -INFINITY;
}

template <typename Tin>
static int launch_simt_t(const AttnParams& p, cudaStream_t stream) {
  const long long rows = (long long)p.B * p.N * p.H;
  const unsigned grid = (unsigned)((rows + kSimtWarps - 1) / kSimtWarps);
  const int d_qk = p.d_l + p.d_r;
  const int pl = ceil_div(d_qk, 32);
  if (pl <= 4)
    return launch_pdl(attn_simt_kernel<Tin, 4>, grid, 32 * kSimtWarps, 0, stream, p);
  else if (pl <= 8)
    return launch_pdl(attn_simt_kernel<Tin, 8>, grid, 32 * kSimtWarps, 0, stream, p);
  else if (pl <= 18)
    return launch_pdl(attn_simt_kernel<Tin, 18>, grid, 32 * kSimtWarps, 0, stream, p);
  else
    return launch_pdl(attn_simt_kernel<Tin, kMaxPerLane>, grid, 32 * kSimtWarps, 0, stream, p);
}

int launch_attn_simt(const AttnParams& p, cudaStream_t stream) {
  if (p.in_dtype == DDT_F32) return launch_simt_t<float>(p, stream);
  return launch_simt_t<uint16_t>(p, stream);
}

}  // namespace ddt
