// Tensor-core tree-verify attention for bf16 inputs with the Kimi K2.6 MLA
// shape (512-d latent + 64-d RoPE; 576-d QK, 512-d V), sm_100a.
//
// What it computes is fixed in ddt.h (ddt_verify_attn): every tree node's
// head attends, in absorbed-MLA form, to the request's committed latent rows
// plus the tree rows its visibility mask selects
// ("autoregressive_test_driver_kdtree_engine", section "The Broader Context":
// tree-verify MLA-absorb attention with visibility masking).
//
// Structure (one unit = 128 query rows x one slice of the request's keys):
//  * A CTA pair (cluster of 2) owns a unit. tcgen05 MMAs run with
//    cta_group::2 and M = 128: each CTA feeds 64 query rows, and its tensor
//    memory holds those 64 rows with the N columns split across lane halves.
//    That halves every accumulator's TMEM footprint, so one CTA keeps two S
//    buffers (2 x 128 columns) and the full 64 x 512 fp32 output (256
//    columns) resident at once; with a single CTA the 128 x 512 output alone
//    would fill all 512 columns.
//  * Key tiles are 256 keys. QK: N = 256 keys (each CTA supplies 128 keys'
//    576-d rows through TMA), K-steps of 16 over 576 dims. PV: two MMAs with
//    N = 256 output dims each (each CTA supplies 128 dims of the latent rows,
//    read MN-major from the same TMA tile layout), K = 256 keys.
//  * Both rings hand the tensor pipe 8 MMAs per stage release: a
//    tcgen05.commit or an mbarrier wait in an issuing thread costs the pipe
//    up to ~90 ns unless enough MMAs are queued around it.
//  * Warp roles per CTA: warps 0 / 2 = TMA producers of the QK ring (query
//    and key chunks; the query is re-streamed with every key tile so shared
//    memory holds deeper rings) and of the value ring (both CTAs load their
//    halves into their own shared memory, completion counted on the leader
//    CTA's barriers), warps 1 / 3 = the QK and PV MMA issuers (leader CTA
//    only; warp 1 also allocates TMEM),
//    warps 4..11 = softmax (TMEM lane quarter = warp % 4, two warps per
//    quarter; thread = one query row x one 64-key group of the tile, and one
//    of the row's two 128-dim output accumulator blocks).
//  * Two issuing threads because every mbarrier wait in an issuing thread
//    stalls the tensor pipe for about as long as two MMAs (its issue queue
//    is shallow); with QK and PV on separate threads and separate rings, one
//    thread's waits hide behind the other's MMAs.
//  * Online softmax in the base-2 domain; the running max is only moved (and
//    the TMEM output rescaled) when it grows by more than 8, so P <= 256.
//    P is rounded to bf16 into shared memory (K-major, 128-byte swizzle) and
//    fed to the PV MMA. The tree part of the keys is masked per row with the
//    node's ancestor bitmask; key groups that run past the request's last key
//    are loaded from a window that ends at that key (never outside the
//    request's finite rows) and the duplicated keys are masked.
//  * A request's keys can be split into several units (flash-decoding); each
//    split writes unnormalised fp32 partials (O, running max, sum) and a small
//    combine kernel merges them. With one split the kernel writes the final
//    output and lse directly.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include "ddt_kernels.cuh"
#include "sm100_ptx.cuh"

namespace ddt {
namespace tc {

using namespace sm100;

constexpr int kDL = 512, kDR = 64, kDQK = 576;
constexpr int kChunks = kDQK / 64;          // 9 column chunks of 64 (128 bytes)
constexpr int kTileKeys = 256;              // keys per tile
constexpr int kBoxBytes = 8192;
constexpr int kPBytes = 4 * kBoxBytes;        // 64 rows x 256 keys bf16
constexpr int kMaxW = 8;                      // mask words per row (N <= 256)
constexpr int kSoftmaxWarps = 8;               // warps 4..11, two per SM sub-partition
constexpr int kThreads = 32 * (4 + kSoftmaxWarps);
constexpr float kRescaleThreshold = 8.0f;     // log2 units

// shared memory map (bytes from the 1024-aligned base)
// QK ring: one stage = this CTA's Q chunk (64 rows x 64 dims, 8 KB) + K chunk
// (128 keys x 64 dims, 16 KB); stages are released in pairs (8 MMAs / commit).
// V ring: one stage = 64 keys x both 128-dim output blocks (4 boxes, 32 KB).
constexpr int kKStages = 4;
constexpr int kKStageBytes = 3 * kBoxBytes;    // 24 KB
constexpr int kVStages = 2;
constexpr int kVStageBytes = 4 * kBoxBytes;    // 32 KB
constexpr int kOffKRing = 0;
constexpr int kOffVRing = kOffKRing + kKStages * kKStageBytes;
constexpr int kOffP = kOffVRing + kVStages * kVStageBytes;
constexpr int kOffMisc = kOffP + kPBytes;
// misc: barriers (8 B each)
constexpr int kBarKFull = 0;                          // [kKStages / 2] leader: TMA bytes of a stage pair, both CTAs
constexpr int kBarKEmpty = kBarKFull + kKStages / 2;  // [kKStages / 2] each CTA: QK MMAs done with a stage pair
constexpr int kBarVFull = kBarKEmpty + kKStages / 2;  // [kVStages]
constexpr int kBarVEmpty = kBarVFull + kVStages;      // [kVStages]
constexpr int kBarSFull = kBarVEmpty + kVStages;      // [2] each CTA: S buffer written
constexpr int kBarSEmpty = kBarSFull + 2;             // [2] leader: S buffer read (softmax warps of both CTAs)
constexpr int kBarPFull = kBarSEmpty + 2;             // leader: P written (softmax warps of both CTAs)
constexpr int kBarOFull = kBarPFull + 1;              // each CTA: PV finished
constexpr int kNumBars = kBarOFull + 1;
constexpr int kOffRed = kOffMisc + 256;                 // float [2 parity][4 groups][64]
constexpr int kOffLred = kOffRed + 2 * 4 * 64 * 4;      // float [4][64]
constexpr int kOffMask = kOffLred + 4 * 64 * 4;         // uint32 [64][kMaxW]
constexpr int kOffTmem = kOffMask + 64 * kMaxW * 4;     // uint32
constexpr int kSmemBytes = kOffTmem + 16;
constexpr int kSmemAlloc = kSmemBytes + 1024;           // slack for 1024 alignment
static_assert(kNumBars * 8 <= 256, "barrier area");
static_assert(kKStages % 2 == 0, "QK stages are released in pairs");
static_assert(kSmemAlloc <= 232448, "shared memory budget");

// TMEM columns
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO0 = 256, kColO1 = 384;

constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 256, false, false);
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 256, false, true);

struct TcParams {
  const int64_t* cache_off;
  const int32_t* cache_len;
  const uint32_t* mask;
  const int32_t* n_nodes;
  int B, N, H, W;
  float scale_log2;  // scale * log2(e)
  int splits;
  int rowtiles;      // per request: ceil(N * H / 128)
  int out_dtype;
  void* out;
  float* lse;
  float* part_o;     // [splits][B*N*H][512]
  float* part_ml;    // [splits][B*N*H][2]
  int* abort;
};

struct UnitInfo {
  int b, rt, split;
  int off_row;       // first pool row of the request (fits int: checked on host)
  int L, n, nkeys;
  int kb, ke, T;     // key range [kb, ke) of this unit, T tiles
};

__device__ __forceinline__ UnitInfo unit_info(const TcParams& p, int unit) {
  UnitInfo u;
  u.split = unit % p.splits;
  const int t = unit / p.splits;
  u.rt = t % p.rowtiles;
  u.b = t / p.rowtiles;
  u.off_row = (int)p.cache_off[u.b];
  u.L = p.cache_len[u.b];
  u.n = p.n_nodes[u.b];
  u.nkeys = u.L + u.n;
  const int tiles = (u.nkeys + kTileKeys - 1) / kTileKeys;
  const int per = (tiles + p.splits - 1) / p.splits;
  const int t0 = min(tiles, u.split * per);
  const int t1 = min(tiles, t0 + per);
  u.T = t1 - t0;
  u.kb = t0 * kTileKeys;
  u.ke = min(u.nkeys, t1 * kTileKeys);
  // a row tile whose first node is already a pad node has nothing to compute
  const int first_node = (u.rt * 128) / p.H;
  if (u.n <= 0 || first_node >= u.n) u.T = 0;
  return u;
}

// first pool row (relative to the request) that key group g0 is loaded from:
// a full group loads itself, a group that reaches past the last key loads the
// 64 keys that end at the last key (duplicates are masked in the softmax).
__device__ __forceinline__ int group_window(int g0, int nkeys) { return (g0 + 64 <= nkeys) ? g0 : nkeys - 64; }

// 64 bits of a row mask starting at bit t0 (t0 may be negative)
__device__ __forceinline__ uint64_t mask_bits64(const uint32_t* mw, int W, int t0) {
  if (t0 <= -64 || t0 >= W * 32) return 0ull;
  int lo = t0 < 0 ? 0 : t0;
  const int w = lo >> 5, sh = lo & 31;
  uint32_t a = w < W ? mw[w] : 0u, b2 = (w + 1) < W ? mw[w + 1] : 0u, c = (w + 2) < W ? mw[w + 2] : 0u;
  uint64_t lo64 = ((uint64_t)b2 << 32) | a;
  uint64_t v = sh ? ((lo64 >> sh) | ((uint64_t)c << (64 - sh))) : lo64;
  if (t0 < 0) v <<= (-t0);
  return v;
}

__device__ __forceinline__ uint64_t bits_below(int k) {  // bits [0, k), k clamped to [0, 64]
  return k <= 0 ? 0ull : (k >= 64 ? ~0ull : ((1ull << k) - 1ull));
}

// visibility of keys kw + c (c = 0..63) for one row
__device__ __forceinline__ uint64_t group_visibility(int kw, int g0, int kend, int L, const uint32_t* mw, int W) {
  const uint64_t range = bits_below(kend - kw) & ~bits_below(g0 - kw);
  if (range == 0ull) return 0ull;
  const uint64_t cache = bits_below(L - kw);
  if ((range & ~cache) == 0ull) return range;  // all in the committed cache
  return range & (cache | mask_bits64(mw, W, kw - L));
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kv, TcParams p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  pdl_wait();
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int unit = blockIdx.x >> 1;
  const UnitInfo u = unit_info(p, unit);
  const int rows_total = p.B * p.N * p.H;
  const int req_rows = p.N * p.H;
  const int row0 = u.rt * 128 + 64 * (int)rank;  // first request-relative row of this CTA

  auto bar = [&](int i) -> uint32_t { return sbase + kOffMisc + 8u * (uint32_t)i; };

  // ---------------------------------------------------------------- empty unit
  if (u.T == 0) {
    // no keys for these rows: partials get (m = -inf, l = 0, O = 0); with a
    // single split the rows are pad rows (written as zeros / -inf)
    for (int r = threadIdx.x; r < 64; r += kThreads) {
      const int rr = row0 + r;
      if (rr >= req_rows) continue;
      const size_t grow = (size_t)u.b * req_rows + rr;
      if (p.splits > 1) {
        p.part_ml[((size_t)u.split * rows_total + grow) * 2 + 0] = -INFINITY;
        p.part_ml[((size_t)u.split * rows_total + grow) * 2 + 1] = 0.0f;
      } else if (p.lse) {
        p.lse[grow] = -INFINITY;
      }
    }
    for (int e = threadIdx.x; e < 64 * (kDL / 4); e += kThreads) {
      const int r = e / (kDL / 4), c4 = e % (kDL / 4);
      const int rr = row0 + r;
      if (rr >= req_rows) continue;
      const size_t grow = (size_t)u.b * req_rows + rr;
      if (p.splits > 1) {
        reinterpret_cast<float4*>(p.part_o + ((size_t)u.split * rows_total + grow) * kDL)[c4] =
            make_float4(0.f, 0.f, 0.f, 0.f);
      } else if (p.out_dtype == DDT_F32) {
        reinterpret_cast<float4*>(static_cast<float*>(p.out) + grow * kDL)[c4] = make_float4(0.f, 0.f, 0.f, 0.f);
      } else {
        reinterpret_cast<uint2*>(static_cast<uint16_t*>(p.out) + grow * kDL)[c4] = make_uint2(0u, 0u);
      }
    }
    return;
  }

  // ---------------------------------------------------------------- setup
  if (threadIdx.x == 0) {
    for (int s = 0; s < kKStages / 2; ++s) {
      mbar_init(bar(kBarKFull + s), 1);
      mbar_init(bar(kBarKEmpty + s), 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(bar(kBarVFull + s), 1);
      mbar_init(bar(kBarVEmpty + s), 1);
    }
    mbar_init(bar(kBarSFull + 0), 1);
    mbar_init(bar(kBarSFull + 1), 1);
    mbar_init(bar(kBarSEmpty + 0), 2 * kSoftmaxWarps);
    mbar_init(bar(kBarSEmpty + 1), 2 * kSoftmaxWarps);
    mbar_init(bar(kBarPFull), 2 * kSoftmaxWarps);
    mbar_init(bar(kBarOFull), 1);
    fence_mbar_init_cluster();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_kv);
  }
  // masks of this CTA's 64 rows (node = row / H)
  uint32_t* s_mask = reinterpret_cast<uint32_t*>(smem + kOffMask);
  for (int e = threadIdx.x; e < 64 * kMaxW; e += kThreads) {
    const int r = e / kMaxW, w = e % kMaxW;
    const int rr = row0 + r;
    const int node = rr / p.H;
    uint32_t v = 0u;
    if (rr < req_rows && node < p.N && w < p.W) v = p.mask[((size_t)u.b * p.N + node) * p.W + w];
    s_mask[e] = v;
  }
  if (warp == 1) {
    tmem_alloc_pair(sbase + kOffTmem, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + kOffTmem);
  int* abort = p.abort;

  // one ring of 16 KB stages per operand stream, each with its own producer
  // thread and its own MMA-issuing thread: while one issuer waits on a
  // barrier, the other keeps the tensor pipe fed
  struct Ring {
    int slot = 0;
    uint32_t phase = 0;
  };
  if (warp == 0 && lane == 0) {
    // ============================================================ QK producer
    // per tile and 64-dim chunk: this CTA's Q chunk and its 128 keys' chunk
    const uint32_t full0 = map_to_rank(bar(kBarKFull), 0);
    Ring rg;
    const int qrow = u.b * req_rows + row0;
    for (int t = 0; t < u.T; ++t) {
      const int tile0 = u.kb + t * kTileKeys;
      const int y0 = u.off_row + group_window(tile0 + 128 * (int)rank, u.nkeys);
      const int y1 = u.off_row + group_window(tile0 + 128 * (int)rank + 64, u.nkeys);
      bool ok = true;
      for (int ch = 0; ch < kChunks; ++ch) {
        if ((rg.slot & 1) == 0) {
          if (!mbar_wait(bar(kBarKEmpty + (rg.slot >> 1)), rg.phase ^ 1u, abort)) {
            ok = false;
            break;
          }
          // one barrier per stage pair; the pair is always filled completely
          // (the last pair of the unit may get a duplicate stage, see below)
          if (leader) mbar_arrive_expect_tx(bar(kBarKFull + (rg.slot >> 1)), 4u * kKStageBytes);
        }
        const uint32_t dst = sbase + kOffKRing + rg.slot * kKStageBytes;
        const uint32_t fb = full0 + 8u * (uint32_t)(rg.slot >> 1);
        tma_load_2d_pair(dst, &tm_q, ch * 64, qrow, fb);
        tma_load_2d_pair(dst + kBoxBytes, &tm_kv, ch * 64, y0, fb);
        tma_load_2d_pair(dst + 2 * kBoxBytes, &tm_kv, ch * 64, y1, fb);
        if (++rg.slot == kKStages) { rg.slot = 0; rg.phase ^= 1u; }
      }
      if (!ok) break;
    }
    if (rg.slot & 1) {
      // odd number of stages: complete the last pair's byte count with a
      // repeat of the last Q box + key boxes (never consumed)
      const int tile0 = u.kb + (u.T - 1) * kTileKeys;
      const int y0 = u.off_row + group_window(tile0 + 128 * (int)rank, u.nkeys);
      const int y1 = u.off_row + group_window(tile0 + 128 * (int)rank + 64, u.nkeys);
      const uint32_t dst = sbase + kOffKRing + rg.slot * kKStageBytes;
      const uint32_t fb = full0 + 8u * (uint32_t)(rg.slot >> 1);
      tma_load_2d_pair(dst, &tm_q, (kChunks - 1) * 64, qrow, fb);
      tma_load_2d_pair(dst + kBoxBytes, &tm_kv, (kChunks - 1) * 64, y0, fb);
      tma_load_2d_pair(dst + 2 * kBoxBytes, &tm_kv, (kChunks - 1) * 64, y1, fb);
    }
  } else if (warp == 2 && lane == 0) {
    // ============================================================ V producer
    // per tile and 64-key group: this CTA's two 128-dim value blocks
    const uint32_t full0 = map_to_rank(bar(kBarVFull), 0);
    Ring rg;
    const int x = 128 * (int)rank;
    for (int t = 0; t < u.T; ++t) {
      const int tile0 = u.kb + t * kTileKeys;
      bool ok = true;
      for (int g = 0; g < 4; ++g) {
        if (!mbar_wait(bar(kBarVEmpty + rg.slot), rg.phase ^ 1u, abort)) {
          ok = false;
          break;
        }
        if (leader) mbar_arrive_expect_tx(bar(kBarVFull + rg.slot), 2u * kVStageBytes);
        const int y = u.off_row + group_window(tile0 + 64 * g, u.nkeys);
        const uint32_t dst = sbase + kOffVRing + rg.slot * kVStageBytes;
        const uint32_t fb = full0 + 8u * (uint32_t)rg.slot;
        tma_load_2d_pair(dst, &tm_kv, x, y, fb);
        tma_load_2d_pair(dst + kBoxBytes, &tm_kv, x + 64, y, fb);
        tma_load_2d_pair(dst + 2 * kBoxBytes, &tm_kv, x + 256, y, fb);
        tma_load_2d_pair(dst + 3 * kBoxBytes, &tm_kv, x + 320, y, fb);
        if (++rg.slot == kVStages) { rg.slot = 0; rg.phase ^= 1u; }
      }
      if (!ok) break;
    }
  } else if ((warp == 1 || warp == 3) && lane == 0 && leader) {
    // ============================================================ MMA issuers
    bool ok = true;
    Ring rg;
    // stage data comes from TMA (async proxy to async proxy): the mbarrier
    // wait alone orders it before the MMAs, no tcgen05 fence needed
    if (warp == 1) {
      // Q.K^T into the two S buffers
      for (int t = 0; t < u.T && ok; ++t) {
        const int sb = t & 1;
        if (t >= 2) {
          if (!mbar_wait(bar(kBarSEmpty + sb), (uint32_t)(((t >> 1) + 1) & 1), abort)) { ok = false; break; }
          tc_fence_after();
        }
        const uint32_t d = tmem + (sb ? kColS1 : kColS0);
        for (int ch = 0; ch < kChunks; ++ch) {
          if ((rg.slot & 1) == 0 && !mbar_wait(bar(kBarKFull + (rg.slot >> 1)), rg.phase, abort)) { ok = false; break; }
          const uint32_t a0 = sbase + kOffKRing + rg.slot * kKStageBytes;
          const uint32_t b0 = a0 + kBoxBytes;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_pair_ss(d, smem_desc_sw128(a0 + 32 * k, 16, 1024), smem_desc_sw128(b0 + 32 * k, 16, 1024), kIdescQK,
                        (ch | k) != 0);
          if (rg.slot & 1) mma_commit_pair_mc(bar(kBarKEmpty + (rg.slot >> 1)), 0x3);
          if (++rg.slot == kKStages) { rg.slot = 0; rg.phase ^= 1u; }
        }
        if (ok) mma_commit_pair_mc(bar(kBarSFull + sb), 0x3);
      }
    } else {
      // P.V into the two 128-column output blocks
      for (int t = 0; t < u.T && ok; ++t) {
        if (!mbar_wait(bar(kBarPFull), (uint32_t)(t & 1), abort)) { ok = false; break; }
        tc_fence_after();
        for (int g = 0; g < 4; ++g) {
          if (!mbar_wait(bar(kBarVFull + rg.slot), rg.phase, abort)) { ok = false; break; }
          const uint32_t a0 = sbase + kOffP + g * kBoxBytes;
          const uint32_t b0 = sbase + kOffVRing + rg.slot * kVStageBytes;
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const uint32_t d = tmem + (j ? kColO1 : kColO0);
#pragma unroll
            for (int k = 0; k < 4; ++k)
              mma_pair_ss(d, smem_desc_sw128(a0 + 32 * k, 16, 1024),
                          smem_desc_sw128(b0 + 2 * j * kBoxBytes + 2048 * k, kBoxBytes, 1024), kIdescPV,
                          (t > 0 || g > 0 || k > 0) ? 1u : 0u);
          }
          mma_commit_pair_mc(bar(kBarVEmpty + rg.slot), 0x3);
          if (++rg.slot == kVStages) { rg.slot = 0; rg.phase ^= 1u; }
        }
        if (ok) mma_commit_pair_mc(bar(kBarOFull), 0x3);
      }
    }
  } else if (warp >= 4) {
    // ============================================================ softmax
    // warp w reads TMEM lane quarter w % 4; lane l holds one row (l % 64) and
    // one half of the tile's keys / output dims (l / 64); the two warps of a
    // quarter split that half again (sub): each thread owns one 64-key group
    // of S / P and one of the two 128-column output accumulators.
    const int q4 = warp & 3;
    const int sub = (warp - 4) >> 2;
    const int l = 32 * q4 + lane;          // TMEM lane
    const int rho = l & 63, eta = l >> 6;  // row within CTA, key / dim half
    const int grp = 2 * eta + sub;         // 64-key group of the tile (= P chunk)
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * q4) << 16);
    const uint32_t o_col = sub ? kColO1 : kColO0;
    const uint32_t* mw = s_mask + rho * kMaxW;
    float* red = reinterpret_cast<float*>(smem + kOffRed);
    float* lred = reinterpret_cast<float*>(smem + kOffLred);
    const uint32_t sempty0 = map_to_rank(bar(kBarSEmpty), 0);
    const uint32_t pfull0 = map_to_rank(bar(kBarPFull), 0);
    unsigned char* pchunk = smem + kOffP + grp * kBoxBytes + rho * 128;
    const float sl2 = p.scale_log2;
    float m_used = -INFINITY, lsum = 0.0f;
    bool ok = true;
    // every thread runs all T iterations (and so every named barrier) even
    // after an aborted wait; later waits then return at once
    for (int t = 0; t < u.T; ++t) {
      const int sb = t & 1;
      if (ok && !mbar_wait(bar(kBarSFull + sb), (uint32_t)((t >> 1) & 1), abort)) ok = false;
      tc_fence_after();
      float s[64];
      {
        uint32_t r0[32], r1[32];
        const uint32_t a = lane_addr + (sb ? kColS1 : kColS0) + 64 * sub;
        tmem_ld32(a, r0);
        tmem_ld32(a + 32, r1);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          s[i] = __uint_as_float(r0[i]);
          s[32 + i] = __uint_as_float(r1[i]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader) mbar_arrive_local(bar(kBarSEmpty + sb));
        else mbar_arrive_cluster(sempty0 + 8u * (uint32_t)sb);
      }
      // visibility of this thread's 64 keys; the common case (all committed
      // cache keys, none cut by the unit's range) needs no per-key work
      const int g0 = u.kb + t * kTileKeys + 64 * grp;
      const int kw = group_window(g0, u.nkeys);
      const uint64_t vis = group_visibility(kw, g0, u.ke, u.L, mw, p.W);
      float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
      if (vis == ~0ull) {
#pragma unroll
        for (int c = 0; c < 64; c += 4) {
          mx0 = fmaxf(mx0, s[c]);
          mx1 = fmaxf(mx1, s[c + 1]);
          mx2 = fmaxf(mx2, s[c + 2]);
          mx3 = fmaxf(mx3, s[c + 3]);
        }
      } else {
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const float v = ((vis >> c) & 1ull) ? s[c] : -INFINITY;
          s[c] = v;
          if ((c & 3) == 0) mx0 = fmaxf(mx0, v);
          if ((c & 3) == 1) mx1 = fmaxf(mx1, v);
          if ((c & 3) == 2) mx2 = fmaxf(mx2, v);
          if ((c & 3) == 3) mx3 = fmaxf(mx3, v);
        }
      }
      const float mloc = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * sl2;  // scale > 0 keeps the max
      float* rt = red + sb * 4 * 64;
      rt[grp * 64 + rho] = mloc;
      named_bar_sync(1, 32 * kSoftmaxWarps);
      const float mtile = fmaxf(fmaxf(rt[rho], rt[64 + rho]), fmaxf(rt[128 + rho], rt[192 + rho]));
      const float m_new = fmaxf(m_used, mtile);
      bool rescale = false;
      float alpha = 1.0f;
      if (m_used == -INFINITY) {
        m_used = m_new;  // output is still exactly zero: nothing to rescale
      } else if (m_new > m_used + kRescaleThreshold) {
        alpha = exp2f(m_used - m_new);
        m_used = m_new;
        rescale = true;
      }
      const float mref = (m_used == -INFINITY) ? 0.0f : m_used;
      // probabilities (p = 2^(s * scale * log2e - m)), row sum, bf16 pack
      uint32_t pk[32];
      float ps0 = 0.0f, ps1 = 0.0f;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float p0 = exp2f(fmaf(s[2 * i], sl2, -mref));
        const float p1 = exp2f(fmaf(s[2 * i + 1], sl2, -mref));
        ps0 += p0;
        ps1 += p1;
        __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
        pk[i] = *reinterpret_cast<uint32_t*>(&h2);
      }
      lsum = lsum * alpha + (ps0 + ps1);
      // the P buffer and the output accumulator are free once PV(t-1) is done
      if (t > 0) {
        if (ok && !mbar_wait(bar(kBarOFull), (uint32_t)((t - 1) & 1), abort)) ok = false;
        tc_fence_after();
      }
      if (rescale) {
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          const uint32_t a = lane_addr + o_col + 32 * c;
          tmem_ld32(a, r);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
          tmem_st32(a, r);
        }
        tmem_wait_st();
      }
      // P row segment: 64 keys = 8 x 16 bytes, 128-byte swizzle
#pragma unroll
      for (int u16 = 0; u16 < 8; ++u16) {
        const int pos = u16 ^ (rho & 7);
        *reinterpret_cast<uint4*>(pchunk + pos * 16) =
            make_uint4(pk[4 * u16 + 0], pk[4 * u16 + 1], pk[4 * u16 + 2], pk[4 * u16 + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader) mbar_arrive_local(bar(kBarPFull));
        else mbar_arrive_cluster(pfull0);
      }
    }
    // ---------------------------------------------------------- epilogue
    if (ok) ok = mbar_wait(bar(kBarOFull), (uint32_t)((u.T - 1) & 1), abort);
    tc_fence_after();
    lred[grp * 64 + rho] = lsum;
    named_bar_sync(1, 32 * kSoftmaxWarps);
    const float ltot = (lred[rho] + lred[64 + rho]) + (lred[128 + rho] + lred[192 + rho]);
    const int rr = row0 + rho;
    const bool in_range = rr < req_rows;
    const bool real_row = ok && in_range && (rr / p.H) < u.n;
    // single split: pad rows of a computed tile are written as zeros
    const bool write_row = p.splits > 1 ? real_row : in_range;
    const size_t grow = (size_t)u.b * req_rows + rr;
    const float inv = !real_row ? 0.0f : ((p.splits == 1 && ltot > 0.0f) ? 1.0f / ltot : 1.0f);
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      uint32_t r[32];
      tmem_ld32(lane_addr + o_col + 32 * c, r);
      tmem_wait_ld();
      if (!write_row) continue;
      const int d0 = 256 * sub + 128 * eta + 32 * c;  // first output dim of this chunk
      if (p.splits > 1) {
        float4* dst = reinterpret_cast<float4*>(p.part_o + ((size_t)u.split * rows_total + grow) * kDL + d0);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          dst[i] = make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                               __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
      } else if (p.out_dtype == DDT_F32) {
        float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + grow * kDL + d0);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          dst[i] = make_float4(__uint_as_float(r[4 * i]) * inv, __uint_as_float(r[4 * i + 1]) * inv,
                               __uint_as_float(r[4 * i + 2]) * inv, __uint_as_float(r[4 * i + 3]) * inv);
      } else {
        uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + grow * kDL + d0);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          uint32_t w[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(r[8 * i + 2 * k]) * inv,
                                                      __uint_as_float(r[8 * i + 2 * k + 1]) * inv);
            w[k] = *reinterpret_cast<uint32_t*>(&h2);
          }
          dst[i] = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    }
    if (write_row && grp == 0) {
      if (p.splits > 1) {
        p.part_ml[((size_t)u.split * rows_total + grow) * 2 + 0] = m_used;
        p.part_ml[((size_t)u.split * rows_total + grow) * 2 + 1] = ltot;
      } else if (p.lse) {
        p.lse[grow] = (real_row && ltot > 0.0f) ? (m_used + log2f(ltot)) * 0.6931471805599453f : -INFINITY;
      }
    }
  }
  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

// Merge split partials: O = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s.
__global__ void __launch_bounds__(128) attn_combine_kernel(TcParams p) {
  pdl_wait();
  pdl_launch_dependents();
  const int rows_total = p.B * p.N * p.H;
  const int row = blockIdx.x;
  if (row >= rows_total) return;
  const int b = row / (p.N * p.H);
  const int node = (row / p.H) % p.N;
  const bool real_row = node < p.n_nodes[b];
  float M = -INFINITY;
  for (int s = 0; s < p.splits; ++s) M = fmaxf(M, p.part_ml[((size_t)s * rows_total + row) * 2]);
  float wsum = 0.0f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  const int c4 = threadIdx.x;  // 128 threads x 4 dims
  if (real_row && M != -INFINITY) {
    for (int s = 0; s < p.splits; ++s) {
      const float m = p.part_ml[((size_t)s * rows_total + row) * 2];
      if (m == -INFINITY) continue;
      const float w = exp2f(m - M);
      wsum += w * p.part_ml[((size_t)s * rows_total + row) * 2 + 1];
      const float4 o = reinterpret_cast<const float4*>(p.part_o + ((size_t)s * rows_total + row) * kDL)[c4];
      acc.x += w * o.x; acc.y += w * o.y; acc.z += w * o.z; acc.w += w * o.w;
    }
  }
  const float inv = wsum > 0.0f ? 1.0f / wsum : 0.0f;
  acc.x *= inv; acc.y *= inv; acc.z *= inv; acc.w *= inv;
  if (p.out_dtype == DDT_F32) {
    reinterpret_cast<float4*>(static_cast<float*>(p.out) + (size_t)row * kDL)[c4] = acc;
  } else {
    __nv_bfloat162 a = __floats2bfloat162_rn(acc.x, acc.y), bq = __floats2bfloat162_rn(acc.z, acc.w);
    reinterpret_cast<uint2*>(static_cast<uint16_t*>(p.out) + (size_t)row * kDL)[c4] =
        make_uint2(*reinterpret_cast<uint32_t*>(&a), *reinterpret_cast<uint32_t*>(&bq));
  }
  if (p.lse && threadIdx.x == 0)
    p.lse[row] = (real_row && wsum > 0.0f) ? (M + log2f(wsum)) * 0.6931471805599453f : -INFINITY;
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }
  return fn;
}

static bool make_map(CUtensorMap* m, const void* base, uint64_t rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)kDQK, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)kDQK * 2};
  cuuint32_t box[2] = {64, 64};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// number of key splits: minimise an estimate of the makespan over 74 CTA pairs
static int choose_splits(int B, int N, int H, int max_cache_len) {
  const int rowtiles = (N * H + 127) / 128;
  const int units1 = B * rowtiles;
  const int tiles = (max_cache_len + N + kTileKeys - 1) / kTileKeys;
  const int slots = 74;
  int best = 1;
  double best_t = 1e30;
  for (int s = 1; s <= std::min(16, std::max(1, tiles)); ++s) {
    const int per = (tiles + s - 1) / s;
    const long units = (long)units1 * s;
    const long waves = (units + slots - 1) / slots;
    const double t = (double)waves * (per + 0.6) + (s > 1 ? 0.4 : 0.0);
    if (t < best_t - 1e-9) { best_t = t; best = s; }
  }
  return best;
}

static size_t ws_header() { return 256; }

}  // namespace tc

bool tc_attn_supported(int d_l, int d_r, int in_dtype) {
  return in_dtype == DDT_BF16 && d_l == tc::kDL && d_r == tc::kDR;
}

size_t tc_attn_workspace_bytes(int B, int N, int H, int max_cache_len) {
  const int s = tc::choose_splits(B, N, H, max_cache_len);
  size_t bytes = tc::ws_header();
  if (s > 1) {
    const size_t rows = (size_t)B * N * H;
    bytes += (size_t)s * rows * tc::kDL * 4 + (size_t)s * rows * 2 * 4;
  }
  return bytes;
}

int launch_attn_tc(const AttnParams& a, int64_t kv_rows, int max_cache_len, void* workspace, size_t workspace_bytes,
                   cudaStream_t stream) {
  using namespace tc;
  if (a.N > 32 * kMaxW) return DDT_ERR_UNSUPPORTED;
  if (kv_rows > 0x7fffffffLL) return DDT_ERR_UNSUPPORTED;
  const long long q_rows = (long long)a.B * a.N * a.H;
  if (q_rows > 0x7fffffffLL) return DDT_ERR_UNSUPPORTED;
  CUtensorMap tq, tkv;
  if (!make_map(&tq, a.q, (uint64_t)q_rows) || !make_map(&tkv, a.kv, (uint64_t)kv_rows)) return DDT_ERR_CUDA;
  TcParams p{};
  p.cache_off = a.cache_off;
  p.cache_len = a.cache_len;
  p.mask = a.mask;
  p.n_nodes = a.n_nodes;
  p.B = a.B;
  p.N = a.N;
  p.H = a.H;
  p.W = a.W;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.splits = choose_splits(a.B, a.N, a.H, max_cache_len);
  p.rowtiles = (a.N * a.H + 127) / 128;
  p.out_dtype = a.out_dtype;
  p.out = a.out;
  p.lse = a.lse;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  p.abort = reinterpret_cast<int*>(ws);
  if (p.splits > 1) {
    const size_t rows = (size_t)a.B * a.N * a.H;
    p.part_o = reinterpret_cast<float*>(ws + ws_header());
    p.part_ml = reinterpret_cast<float*>(ws + ws_header() + (size_t)p.splits * rows * kDL * 4);
  }
  if (workspace_bytes < tc_attn_workspace_bytes(a.B, a.N, a.H, max_cache_len)) return DDT_ERR_INVALID_ARG;
  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc) != cudaSuccess)
      return DDT_ERR_CUDA;
    attr_set = true;
  }
  const long long units = (long long)a.B * p.rowtiles * p.splits;
  int st = launch_pdl(attn_tc_kernel, (unsigned)(2 * units), kThreads, kSmemAlloc, stream, tq, tkv, p);
  if (st != DDT_OK || p.splits == 1) return st;
  return launch_pdl(attn_combine_kernel, (unsigned)q_rows, 128, 0, stream, p);
}

}  // namespace ddt
