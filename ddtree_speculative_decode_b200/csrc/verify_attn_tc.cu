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
//  * The CTA's 64 query rows (72 KB) are loaded once per unit and stay in
//    shared memory. Each ring stage feeds 4 MMAs and is released on its own
//    (the QK ring: this CTA's 128 keys of one 64-dim chunk; the V ring: 64
//    keys x one 128-dim block of each output half), so most of each ring is
//    in flight at any time. Re-streaming the Q chunk with every key chunk
//    instead (a fourth of the bytes every tile moves from L2) measured 3 %
//    slower on the long-context workload.
//  * Three issuing threads because every mbarrier wait in an issuing thread
//    stalls the tensor pipe for about as long as two MMAs (its issue queue
//    is shallow): QK on one, and PV on one per 256-column output block (the
//    two blocks are separate accumulators, each fed by the V ring's slots of
//    one parity), so one thread's waits hide behind the others' MMAs.
//  * Online softmax in the base-2 domain; the running max is only moved (and
//    the TMEM output rescaled) when it grows by more than 8, so P <= 256.
//    P is rounded to bf16 into shared memory (K-major, 128-byte swizzle) and
//    fed to the PV MMA. The tree part of the keys is masked per row with the
//    node's ancestor bitmask; key groups that run past the request's last key
//    are loaded from a window that ends at that key (never outside the
//    request's finite rows) and the duplicated keys are masked.
//  * The kernel may start while the tree build (the kernel before it) still
//    runs: a unit's key range is planned over cache_len + N, its committed-
//    cache tiles need nothing from the build, and each role waits for the
//    build only when it first needs the tree (unit_tree).
//  * A request's keys can be split into several units (flash-decoding); each
//    split writes unnormalised fp32 partials (O, running max, sum) and counts
//    its arrival per (row tile, CTA half); the split that arrives last merges
//    the partials into the final output. With one split the kernel writes the
//    final output and lse directly.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "ddt_kernels.cuh"
#include "sm100_ptx.cuh"

namespace ddt {
namespace tc {

using namespace sm100;

constexpr int kDL = 512, kDR = 64, kDQK = 576;
constexpr int kChunks = kDQK / 64;          // 9 column chunks of 64 (128 bytes)
constexpr int kTileKeys = 256;              // keys per tile
constexpr int kMaxSplits = 16;  // key splits per request at most
constexpr int kBoxBytes = 8192;
constexpr int kPBytes = 4 * kBoxBytes;        // 64 rows x 256 keys bf16
constexpr int kMaxW = 8;                      // mask words per row (N <= 256)
constexpr int kSoftmaxWarps = 8;               // warps 4..11, two per SM sub-partition
constexpr int kPV1Warp = 4 + kSoftmaxWarps;           // warp 12: the second P.V issuer
constexpr int kThreads = 32 * (5 + kSoftmaxWarps);
constexpr float kRescaleThreshold = 8.0f;     // log2 units

// shared memory map (bytes from the 1024-aligned base)
// Q: the CTA's 64 rows as 9 boxes of 64 dims (72 KB), loaded once per unit.
// QK ring: one stage = this CTA's K chunk (128 keys x 64 dims, 16 KB).
// V ring: one stage = 64 keys x this CTA's 128-dim block of one output half
// (2 boxes, 16 KB).
constexpr int kQBytes = kChunks * kBoxBytes;   // 72 KB: the CTA's 64 query rows, resident for the unit
constexpr int kKStages = 3;
constexpr int kKStageBytes = 2 * kBoxBytes;    // 16 KB: the CTA's 128 keys of one 64-dim chunk
constexpr int kKGroup = 1;                     // QK stages released together (one barrier each way)
constexpr int kKBars = kKStages / kKGroup;
constexpr int kVStages = 4;
constexpr int kVStageBytes = 2 * kBoxBytes;    // 16 KB: 64 keys x one 128-dim block of each output half
constexpr int kOffQ = 0;
constexpr int kOffKRing = kOffQ + kQBytes;
constexpr int kOffVRing = kOffKRing + kKStages * kKStageBytes;
constexpr int kOffP = kOffVRing + kVStages * kVStageBytes;
constexpr int kOffMisc = kOffP + kPBytes;
// misc: barriers (8 B each)
constexpr int kBarKFull = 0;                          // [kKBars] leader: TMA bytes of a stage group, both CTAs
constexpr int kBarKEmpty = kBarKFull + kKBars;        // [kKBars] each CTA: QK MMAs done with a stage group
constexpr int kBarVFull = kBarKEmpty + kKBars;        // [kVStages]
constexpr int kBarVEmpty = kBarVFull + kVStages;      // [kVStages]
constexpr int kBarSFull = kBarVEmpty + kVStages;      // [2] each CTA: S buffer written
constexpr int kBarSEmpty = kBarSFull + 2;             // [2] leader: S buffer read (softmax warps of both CTAs)
constexpr int kBarPFull = kBarSEmpty + 2;             // leader: P written (softmax warps of both CTAs)
constexpr int kBarOFull = kBarPFull + 1;              // each CTA: PV finished
constexpr int kBarEpi = kBarOFull + 1;                // [4] each CTA: epilogue tile loads, one per 32-dim chunk
constexpr int kBarXReady = kBarEpi + 4;               // each CTA: the other split's CTA of these rows is done with its MMAs
constexpr int kBarXData = kBarXReady + 1;             // [4] each CTA: the other split's partial, one per 32-dim chunk (bulk copies)
constexpr int kBarQFull = kBarXData + 4;              // leader: the resident Q rows of both CTAs
constexpr int kNumBars = kBarQFull + 1;
constexpr int kOffRed = kOffMisc + 256;                 // float [2 parity][4 groups][64]
constexpr int kOffLred = kOffRed + 2 * 4 * 64 * 4;      // float [4][64]
constexpr int kOffMask = kOffLred + 4 * 64 * 4;         // uint32 [64][kMaxW]
constexpr int kOffTmem = kOffMask + 64 * kMaxW * 4;     // uint32
constexpr int kSmemBytes = kOffTmem + 16;
constexpr int kSmemAlloc = kSmemBytes + 1024;           // slack for 1024 alignment
static_assert(kNumBars * 8 <= 256, "barrier area");
static_assert(kKStages % kKGroup == 0, "QK stages are released in whole groups");
static_assert(kSmemAlloc <= 232448, "shared memory budget");
static_assert(kVStages % 2 == 0, "each P.V issuer owns the ring slots of one parity");

// epilogue staging (reuses the rings once the last MMA has completed): the
// CTA's 64 rows x 512 dims as 128-byte-wide boxes of 64 rows, 128B-swizzled,
// fp32 (16 boxes, 128 KB) at kOffStage32 and bf16 (8 boxes, 64 KB) at
// kOffStage16
constexpr int kOffStage32 = 0;
constexpr int kOffStage16 = 16 * kBoxBytes;
static_assert(kOffStage16 + 8 * kBoxBytes <= kOffMisc, "epilogue staging fits in the rings");

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
  int csize;         // CTAs per cluster: 2 (one pair), or 4 (both key splits of a row tile, splits == 2)
  int rowtiles;      // per request: ceil(N * H / 128)
  int out_dtype;
  void* out;
  float* lse;
  float* part_o;     // [splits][B*N*H][512]
  float* part_ml;    // [splits][B*N*H][2]
  unsigned* counter; // [B * rowtiles * 2][2] per (row tile, CTA half): splits done, partials published; zero between calls
  int32_t* dev_status;  // [B], nullable: DDT_OK or DDT_ERR_BOUNDS
  int64_t kv_rows;
  int* abort;        // workspace status word: DDT_ERR_TIMEOUT after a wait gave up
  uint64_t wait_ns;  // wall-clock limit of every wait
};

// A unit's work: its key range is planned over the budget's keys (cache_len
// + N) from inputs the tree build does not write, so a unit can start on its
// committed-cache tiles while the build still runs; the tree's size (and the
// pool-bound check) comes in once a role needs it (unit_tree, after waiting
// for the build).
struct UnitInfo {
  int b, rt, split;
  int off_row;       // first pool row of the request (as an int; a bad offset is caught by unit_tree)
  int L;             // committed keys (cache_len, at least 0)
  int kb, kend_plan; // key range [kb, kend_plan) of this unit over the budget's keys
  int T;             // tiles of the unit
  int tt;            // tiles [0, tt) hold committed keys only (need nothing from the build)
  int active;        // splits of this request that get keys (splits [0, active))
  // set by unit_tree:
  int n, nkeys, ke;  // tree nodes, keys, end of this unit's range over the real keys
  bool oob;          // the request's rows do not lie in the pool: all its rows are pad rows
  bool tree;         // unit_tree has run
};

__device__ __forceinline__ UnitInfo unit_plan(const TcParams& p, int unit) {
  UnitInfo u;
  u.split = unit % p.splits;
  const int t = unit / p.splits;
  u.rt = t % p.rowtiles;
  u.b = t / p.rowtiles;
  const int64_t off = p.cache_off[u.b];
  const int L = p.cache_len[u.b];
  u.off_row = (int)off;
  u.L = max(L, 0);
  const long long nk_plan = (long long)u.L + p.N;
  const long long tiles_ll = (nk_plan + kTileKeys - 1) / kTileKeys;
  const int tiles = (int)(tiles_ll < (1LL << 24) ? tiles_ll : (1LL << 24));
  // splits get floor or ceil(tiles / splits) tiles, the larger shares last
  // (where the request's ragged last tile is); splits past `tiles` get none
  u.active = min(p.splits, tiles);
  const int t0 = u.split < u.active ? (int)((long long)u.split * tiles / u.active) : tiles;
  const int t1 = u.split < u.active ? (int)((long long)(u.split + 1) * tiles / u.active) : tiles;
  u.T = t1 - t0;
  u.kb = t0 * kTileKeys;
  const long long kend = (long long)t1 * kTileKeys;
  u.kend_plan = (int)(nk_plan < kend ? nk_plan : kend);
  u.tt = u.L > u.kb ? min(u.T, (u.L - u.kb) / kTileKeys) : 0;
  u.n = 0;
  u.nkeys = u.L;
  u.ke = min(u.L, u.kend_plan);
  u.oob = false;
  u.tree = false;
  return u;
}

// The tree's part: wait for the build (programmatic launch: its writes are
// visible after the wait), then the node count and the pool-bound check. A
// request whose rows do not lie in the pool keeps the plan's loads (TMA
// returns zeros outside the pool) and is written as pad rows.
__device__ __forceinline__ void unit_tree(const TcParams& p, UnitInfo& u) {
  if (u.tree) return;
  pdl_wait();
  const int64_t off = p.cache_off[u.b];
  const int L = p.cache_len[u.b], n = p.n_nodes[u.b];
  u.oob = n < 0 || n > p.N || off < 0 || L < 0 || off + L + n > p.kv_rows;
  u.n = u.oob ? 0 : n;
  u.nkeys = u.L + u.n;
  u.ke = min(u.nkeys, u.kend_plan);
  u.tree = true;
}

// 2^x with the hardware approximation, subnormal results flushed to zero: the
// probabilities are rounded to bf16 next, and a probability below 2^-126 of
// the row maximum cannot change a bf16 P.V product or the row sum.
__device__ __forceinline__ float ex2_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 64-key groups of the unit's tile t that hold at least one key of the unit
// (the last tile of a request can be ragged: P.V skips its empty groups)
__device__ __forceinline__ int live_groups(const UnitInfo& u, int t) {
  const int tile0 = u.kb + t * kTileKeys;
  return min(4, (u.ke - tile0 + 63) / 64);
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

__device__ __forceinline__ int ld_volatile_gpu(const int* p) {
  int v;
  asm volatile("ld.volatile.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kv,
                   const __grid_constant__ CUtensorMap tm_out, const __grid_constant__ CUtensorMap tm_part, TcParams p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  // no wait for the preceding kernel (the tree build) here: see unit_tree
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // A CTA pair (ranks 2k, 2k + 1 of the cluster) runs one unit with the
  // 2-CTA MMA; a cluster of 4 holds both key splits of one row tile, so the
  // splits merge through distributed shared memory.
  const uint32_t crank = cluster_ctarank();
  const uint32_t rank = crank & 1u;    // CTA within its pair
  const uint32_t pbase = crank & ~1u;  // cluster rank of the pair's leader CTA
  const bool leader = rank == 0;
  const uint16_t pmask = (uint16_t)(0x3u << pbase);
  const int unit = p.csize == 4 ? (int)((blockIdx.x >> 2) * 2 + (crank >> 1)) : (int)(blockIdx.x >> 1);
  UnitInfo u = unit_plan(p, unit);
  const int rows_total = p.B * p.N * p.H;
  const int req_rows = p.N * p.H;
  const int row0 = u.rt * 128 + 64 * (int)rank;  // first request-relative row of this CTA

  auto bar = [&](int i) -> uint32_t { return sbase + kOffMisc + 8u * (uint32_t)i; };

  // ---------------------------------------------------------------- empty unit
  // a split past the last one that gets keys has nothing to do (in a 4-CTA
  // cluster an idle pair still takes part in the cluster-wide barriers
  // below); pad rows of real units are written as zeros by their epilogue.
  // this CTA's 64 rows as pad rows (zeros, lse -inf), all threads
  auto write_pad_rows = [&]() {
    for (int r = threadIdx.x; r < 64; r += kThreads) {
      const int rr = row0 + r;
      if (rr >= req_rows) continue;
      const size_t grow = (size_t)u.b * req_rows + rr;
      if (p.lse) p.lse[grow] = -INFINITY;
    }
    for (int e = threadIdx.x; e < 64 * (kDL / 4); e += kThreads) {
      const int r = e / (kDL / 4), c4 = e % (kDL / 4);
      const int rr = row0 + r;
      if (rr >= req_rows) continue;
      const size_t grow = (size_t)u.b * req_rows + rr;
      if (p.out_dtype == DDT_F32) {
        reinterpret_cast<float4*>(static_cast<float*>(p.out) + grow * kDL)[c4] = make_float4(0.f, 0.f, 0.f, 0.f);
      } else {
        reinterpret_cast<uint2*>(static_cast<uint16_t*>(p.out) + grow * kDL)[c4] = make_uint2(0u, 0u);
      }
    }
  };
  const bool idle = u.T == 0;
  if (idle && p.csize == 2) return;

  // ---------------------------------------------------------------- setup
  if (threadIdx.x == 0) {
    for (int s = 0; s < kKBars; ++s) {
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
    mbar_init(bar(kBarOFull), 2);
    for (int c = 0; c < 4; ++c) mbar_init(bar(kBarEpi + c), 1);
    mbar_init(bar(kBarXReady), kSoftmaxWarps);
    mbar_init(bar(kBarQFull), 1);
    for (int c = 0; c < 4; ++c) mbar_init(bar(kBarXData + c), 1);
    fence_mbar_init_cluster();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_kv);
  }
  // masks of this CTA's 64 rows (node = row / H): loaded by the softmax
  // threads once the build is done (the first tile that reaches tree keys)
  uint32_t* s_mask = reinterpret_cast<uint32_t*>(smem + kOffMask);
  if (warp == 1) {
    tmem_alloc_pair(sbase + kOffTmem, 512);
    tmem_relinquish_pair();
  }
  // a workspace whose status word already holds an error (an earlier call
  // gave up a wait) makes the call do no work: one thread of the cluster's
  // first CTA reads the word and every CTA of the cluster takes its value, so
  // the CTAs that share barriers agree
  if (crank == 0 && threadIdx.x == 0) *reinterpret_cast<volatile int*>(smem + kOffTmem + 8) = ld_volatile_gpu(p.abort);
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + kOffTmem);
  const bool aborted = ld_cluster_u32(map_to_rank(sbase + kOffTmem + 8, 0)) != 0u;
  int* abort = p.abort;
  const uint64_t wlim = p.wait_ns;

  // one ring of 16 KB stages per operand stream, each with its own producer
  // thread and its own MMA-issuing threads: while one issuer waits on a
  // barrier, the others keep the tensor pipe fed
  struct Ring {
    int slot = 0;
    uint32_t phase = 0;
  };
  if (idle || aborted) {
    // nothing to compute: straight to the cluster-wide teardown (after an
    // earlier timeout split 0 writes its rows as pad rows)
    if (aborted && !idle && u.split == 0) {
      write_pad_rows();
      if (p.dev_status && u.rt == 0 && rank == 0 && threadIdx.x == 0) p.dev_status[u.b] = DDT_ERR_TIMEOUT;
    }
  } else if (warp == 0 && lane == 0) {
    // ============================================================ QK producer
    // the CTA's Q rows once, then per tile and 64-dim chunk: its 128 keys' chunk
    const uint32_t full0 = map_to_rank(bar(kBarKFull), pbase);
    Ring rg;
    const int qrow = u.b * req_rows + row0;
    {
      const uint32_t qfull = map_to_rank(bar(kBarQFull), pbase);
      if (leader) mbar_arrive_expect_tx(bar(kBarQFull), 2u * kQBytes);
      for (int ch = 0; ch < kChunks; ++ch) tma_load_2d_pair(sbase + kOffQ + ch * kBoxBytes, &tm_q, ch * 64, qrow, qfull);
    }
    for (int t = 0; t < u.T; ++t) {
      if (t >= u.tt) unit_tree(p, u);  // windows of a tile that reaches tree keys depend on the tree's size
      const int tile0 = u.kb + t * kTileKeys;
      const int y0 = u.off_row + group_window(tile0 + 128 * (int)rank, u.nkeys);
      const int y1 = u.off_row + group_window(tile0 + 128 * (int)rank + 64, u.nkeys);
      bool ok = true;
      for (int ch = 0; ch < kChunks; ++ch) {
        if (rg.slot % kKGroup == 0) {
          if (!mbar_wait(bar(kBarKEmpty + rg.slot / kKGroup), rg.phase ^ 1u, abort, wlim)) {
            ok = false;
            break;
          }
          // one barrier per stage group; a group is always filled completely
          // (the last group of the unit may get repeated stages, see below)
          if (leader) mbar_arrive_expect_tx(bar(kBarKFull + rg.slot / kKGroup), 2u * kKGroup * kKStageBytes);
        }
        const uint32_t dst = sbase + kOffKRing + rg.slot * kKStageBytes;
        const uint32_t fb = full0 + 8u * (uint32_t)(rg.slot / kKGroup);
        tma_load_2d_pair(dst, &tm_kv, ch * 64, y0, fb);
        tma_load_2d_pair(dst + kBoxBytes, &tm_kv, ch * 64, y1, fb);
        if (++rg.slot == kKStages) { rg.slot = 0; rg.phase ^= 1u; }
      }
      if (!ok) break;
    }
    while (rg.slot % kKGroup != 0) {
      // a partly filled last group: complete its byte count with repeats of
      // the last Q box + key boxes (never consumed)
      const int tile0 = u.kb + (u.T - 1) * kTileKeys;
      const int y0 = u.off_row + group_window(tile0 + 128 * (int)rank, u.nkeys);
      const int y1 = u.off_row + group_window(tile0 + 128 * (int)rank + 64, u.nkeys);
      const uint32_t dst = sbase + kOffKRing + rg.slot * kKStageBytes;
      const uint32_t fb = full0 + 8u * (uint32_t)(rg.slot / kKGroup);
      tma_load_2d_pair(dst, &tm_kv, (kChunks - 1) * 64, y0, fb);
      tma_load_2d_pair(dst + kBoxBytes, &tm_kv, (kChunks - 1) * 64, y1, fb);
      if (++rg.slot == kKStages) { rg.slot = 0; rg.phase ^= 1u; }
    }
  } else if (warp == 2 && lane == 0) {
    // ============================================================ V producer
    // per tile and 64-key group: this CTA's two 128-dim value blocks
    const uint32_t full0 = map_to_rank(bar(kBarVFull), pbase);
    Ring rg;
    const int x = 128 * (int)rank;
    for (int t = 0; t < u.T; ++t) {
      if (t >= u.tt) unit_tree(p, u);  // live groups and windows of a tile that reaches tree keys
      const int tile0 = u.kb + t * kTileKeys;
      bool ok = true;
      const int ng = live_groups(u, t);
      for (int g = 0; g < ng && ok; ++g) {
        const int y = u.off_row + group_window(tile0 + 64 * g, u.nkeys);
        // one stage per output half j: this CTA's 128 dims of it
        for (int j = 0; j < 2; ++j) {
          if (!mbar_wait(bar(kBarVEmpty + rg.slot), rg.phase ^ 1u, abort, wlim)) {
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(bar(kBarVFull + rg.slot), 2u * kVStageBytes);
          const uint32_t dst = sbase + kOffVRing + rg.slot * kVStageBytes;
          const uint32_t fb = full0 + 8u * (uint32_t)rg.slot;
          tma_load_2d_pair(dst, &tm_kv, x + 256 * j, y, fb);
          tma_load_2d_pair(dst + kBoxBytes, &tm_kv, x + 256 * j + 64, y, fb);
          if (++rg.slot == kVStages) { rg.slot = 0; rg.phase ^= 1u; }
        }
      }
      if (!ok) break;
    }
  } else if ((warp == 1 || warp == 3 || warp == kPV1Warp) && lane == 0 && leader) {
    // ============================================================ MMA issuers
    bool ok = true;
    Ring rg;
    // stage data comes from TMA (async proxy to async proxy): the mbarrier
    // wait alone orders it before the MMAs, no tcgen05 fence needed
    if (warp == 1) {
      // Q.K^T into the two S buffers
      if (!mbar_wait(bar(kBarQFull), 0u, abort, wlim)) ok = false;
      for (int t = 0; t < u.T && ok; ++t) {
        const int sb = t & 1;
        if (t >= 2) {
          if (!mbar_wait(bar(kBarSEmpty + sb), (uint32_t)(((t >> 1) + 1) & 1), abort, wlim)) { ok = false; break; }
          tc_fence_after();
        }
        const uint32_t d = tmem + (sb ? kColS1 : kColS0);
        for (int ch = 0; ch < kChunks; ++ch) {
          if (rg.slot % kKGroup == 0 && !mbar_wait(bar(kBarKFull + rg.slot / kKGroup), rg.phase, abort, wlim)) {
            ok = false;
            break;
          }
          const uint32_t a0 = sbase + kOffKRing + rg.slot * kKStageBytes;
          // descriptors once per stage: +32 bytes per K step is +2 in the address field
          const uint64_t da = smem_desc_sw128(sbase + kOffQ + ch * kBoxBytes, 16, 1024), db = smem_desc_sw128(a0, 16, 1024);
          mma_pair_ss(d, da, db, kIdescQK, ch != 0);
#pragma unroll
          for (int k = 1; k < 4; ++k) mma_pair_ss(d, da + 2 * k, db + 2 * k, kIdescQK, 1u);
          if (rg.slot % kKGroup == kKGroup - 1) mma_commit_pair_mc(bar(kBarKEmpty + rg.slot / kKGroup), pmask);
          if (++rg.slot == kKStages) { rg.slot = 0; rg.phase ^= 1u; }
        }
        if (ok) mma_commit_pair_mc(bar(kBarSFull + sb), pmask);
      }
    } else {
      // P.V into one of the two 128-column output blocks (warp 3: block 0,
      // the second P.V issuer: block 1). The V producer alternates the
      // blocks, so block j's stages are the ring slots of parity j.
      const int j = warp == 3 ? 0 : 1;
      const uint32_t d = tmem + (j ? kColO1 : kColO0);
      rg.slot = j;
      for (int t = 0; t < u.T && ok; ++t) {
        if (!mbar_wait(bar(kBarPFull), (uint32_t)(t & 1), abort, wlim)) { ok = false; break; }
        tc_fence_after();
        if (t >= u.tt) unit_tree(p, u);  // live key groups of a tile that reaches tree keys
        const int ng = live_groups(u, t);
        for (int g = 0; g < ng; ++g) {
          const uint64_t da = smem_desc_sw128(sbase + kOffP + g * kBoxBytes, 16, 1024);
          if (!mbar_wait(bar(kBarVFull + rg.slot), rg.phase, abort, wlim)) { ok = false; break; }
          // +2048 bytes per K step (16 keys) is +128 in the address field
          const uint64_t db = smem_desc_sw128(sbase + kOffVRing + rg.slot * kVStageBytes, kBoxBytes, 1024);
          mma_pair_ss(d, da, db, kIdescPV, (t > 0 || g > 0) ? 1u : 0u);
#pragma unroll
          for (int k = 1; k < 4; ++k) mma_pair_ss(d, da + 2 * k, db + 128 * k, kIdescPV, 1u);
          mma_commit_pair_mc(bar(kBarVEmpty + rg.slot), pmask);
          rg.slot += 2;
          if (rg.slot >= kVStages) { rg.slot -= kVStages; rg.phase ^= 1u; }
        }
        if (ok) mma_commit_pair_mc(bar(kBarOFull), pmask);
      }
    }
  } else if (warp >= 4 && warp < 4 + kSoftmaxWarps) {
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
    const uint32_t sempty0 = map_to_rank(bar(kBarSEmpty), pbase);
    const uint32_t pfull0 = map_to_rank(bar(kBarPFull), pbase);
    unsigned char* pchunk = smem + kOffP + grp * kBoxBytes + rho * 128;
    const float sl2 = p.scale_log2;
    float m_used = -INFINITY, lsum = 0.0f;
    bool ok = true;
    // the tree's part, once: the build's results (node count, pool check)
    // and this CTA's 64 mask rows into shared memory
    auto tree_part = [&]() {
      unit_tree(p, u);
      for (int e = (int)threadIdx.x - 128; e < 64 * kMaxW; e += 32 * kSoftmaxWarps) {
        const int r = e / kMaxW, w = e % kMaxW;
        const int rr = row0 + r;
        const int node = rr / p.H;
        uint32_t v = 0u;
        if (rr < req_rows && node < p.N && w < p.W) v = p.mask[((size_t)u.b * p.N + node) * p.W + w];
        s_mask[e] = v;
      }
      named_bar_sync(1, 32 * kSoftmaxWarps);
    };
    // every thread runs all T iterations (and so every named barrier) even
    // after an aborted wait; later waits then return at once
    for (int t = 0; t < u.T; ++t) {
      if (t == u.tt) tree_part();  // the first tile that reaches tree keys
      const int sb = t & 1;
      if (ok && !mbar_wait(bar(kBarSFull + sb), (uint32_t)((t >> 1) & 1), abort, wlim)) ok = false;
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
      // probabilities (p = 2^(s * scale * log2e - m)), row sum, bf16 pack; the
      // scaling and the sums run on pairs (packed f32x2 FMA and add: the same
      // correctly rounded operations, half the instructions, which matters
      // here because these warps share issue slots with the MMA issuers)
      uint32_t pk[32];
      const float2 sl2v = make_float2(sl2, sl2), nmv = make_float2(-mref, -mref);
      float2 ps = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float2 y = __ffma2_rn(make_float2(s[2 * i], s[2 * i + 1]), sl2v, nmv);
        const float2 pp = make_float2(ex2_ftz(y.x), ex2_ftz(y.y));
        ps = __fadd2_rn(ps, pp);
        __nv_bfloat162 h2 = __floats2bfloat162_rn(pp.x, pp.y);
        pk[i] = *reinterpret_cast<uint32_t*>(&h2);
      }
      lsum = lsum * alpha + (ps.x + ps.y);
      // the P buffer and the output accumulator are free once PV(t-1) is done
      if (t > 0) {
        if (ok && !mbar_wait(bar(kBarOFull), (uint32_t)((t - 1) & 1), abort, wlim)) ok = false;
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
    // O goes from TMEM through swizzled shared-memory boxes to global memory
    // by TMA tile stores, one group of boxes per 32-dim chunk so that staging
    // and storing overlap (rows past the request are clipped by the map).
    //
    // Several key splits: the split that finishes its keys last for these 64
    // rows is the merger. It skips its own partial, waits (bounded) until
    // the other splits -- all already past their keys -- have published
    // theirs, loads them by TMA and merges them into its own O in TMEM:
    //   O = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s,  M = max_s m_s.
    if (ok) ok = mbar_wait(bar(kBarOFull), (uint32_t)((u.T - 1) & 1), abort, wlim);
    tc_fence_after();
    unit_tree(p, u);  // a unit of committed keys only still needs the tree's size for its rows
    if (p.dev_status && u.rt == 0 && u.split == 0 && rank == 0 && threadIdx.x == 128)
      p.dev_status[u.b] = u.oob ? DDT_ERR_BOUNDS : DDT_OK;
    lred[grp * 64 + rho] = lsum;
    const int rr = row0 + rho;
    const bool in_range = rr < req_rows;
    const bool multi = u.active > 1;  // this unit's O is one split's partial
    const size_t grow = (size_t)u.b * req_rows + rr;
    const uint32_t sw = (uint32_t)(rho & 7);
    const bool f32_out = p.out_dtype == DDT_F32;
    int* s_flag = reinterpret_cast<int*>(smem + kOffTmem + 4);
    // both splits of these rows in this cluster: merge through distributed
    // shared memory; otherwise through the workspace (merger elected below)
    const bool xmerge = multi && p.csize == 4;
    const uint32_t xpeer = crank ^ 2u;  // same rows, the other key split
    if (xmerge) {
      // arm the barrier the other split's bulk copy completes on, then tell
      // that CTA that this CTA's staging is free (its MMAs are done)
      if (threadIdx.x == 128 + 128 * (int)(crank >> 1))
        for (int c = 0; c < 4; ++c) mbar_arrive_expect_tx(bar(kBarXData + c), 2u * kBoxBytes + (c == 0 ? 64u * 8u : 0u));
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(map_to_rank(bar(kBarXReady), xpeer));
    }
    unsigned* cnt = (multi && !xmerge) ? p.counter + (((size_t)u.b * p.rowtiles + u.rt) * 2 + rank) * 2 : nullptr;
    if (multi && !xmerge && threadIdx.x == 128) {
      const bool last = atomicAdd(cnt, 1u) == (unsigned)(u.active - 1);
      if (last) cnt[0] = 0u;
      *s_flag = last ? 1 : 0;
    }
    named_bar_sync(1, 32 * kSoftmaxWarps);
    const bool merger = multi && !xmerge && *s_flag != 0;
    const float ltot = (lred[rho] + lred[64 + rho]) + (lred[128 + rho] + lred[192 + rho]);
    const bool real_row = ok && in_range && (rr / p.H) < u.n;
    const float m_own = real_row ? m_used : -INFINITY;
    // 32 values of this thread's row, dims d0.., into the fp32 or bf16 staging
    auto stage_chunk = [&](int d0, const float* f, bool f32) {
      if (f32) {
        unsigned char* row = smem + kOffStage32 + (d0 >> 5) * kBoxBytes + rho * 128;
#pragma unroll
        for (int i = 0; i < 8; ++i)
          *reinterpret_cast<float4*>(row + (((uint32_t)i ^ sw) << 4)) =
              make_float4(f[4 * i], f[4 * i + 1], f[4 * i + 2], f[4 * i + 3]);
      } else {
        unsigned char* row = smem + kOffStage16 + (d0 >> 6) * kBoxBytes + rho * 128;
        const int i0 = (d0 & 63) >> 3;  // 16-byte chunk of the first value
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          uint32_t w[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            __nv_bfloat162 h2 = __floats2bfloat162_rn(f[8 * i + 2 * k], f[8 * i + 2 * k + 1]);
            w[k] = *reinterpret_cast<uint32_t*>(&h2);
          }
          *reinterpret_cast<uint4*>(row + (((uint32_t)(i0 + i) ^ sw) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    };
    // after chunk c is staged by every thread: one thread stores the boxes it
    // completed. kind 0: this split's partial (fp32), 1: final fp32, 2: final
    // bf16 (a bf16 box holds two chunks: stored after odd c)
    auto store_chunk = [&](int c, int kind) {
      if (kind == 2 && !(c & 1)) return;
      fence_proxy_async_smem();
      named_bar_sync(1, 32 * kSoftmaxWarps);
      if (threadIdx.x == 128) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (kind == 0) {
            const int j = 4 * q + c;
            tma_store_4d(&tm_part, sbase + kOffStage32 + j * kBoxBytes, 32 * j, row0, u.b, u.split);
          } else if (kind == 1) {
            const int j = 4 * q + c;
            tma_store_3d(&tm_out, sbase + kOffStage32 + j * kBoxBytes, 32 * j, row0, u.b);
          } else {
            const int j = 2 * q + (c >> 1);
            tma_store_3d(&tm_out, sbase + kOffStage16 + j * kBoxBytes, 64 * j, row0, u.b);
          }
        }
        bulk_commit();
      }
    };
    // TMA loads of split s2's partial rows into the fp32 staging, one barrier per chunk
    auto load_partial = [&](int s2) {
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        mbar_arrive_expect_tx(bar(kBarEpi + c), 4u * kBoxBytes);
        for (int q = 0; q < 4; ++q) {
          const int j = 4 * q + c;
          tma_load_4d(sbase + kOffStage32 + j * kBoxBytes, &tm_part, 32 * j, row0, u.b, s2, bar(kBarEpi + c));
        }
      }
    };
    if (xmerge) {
      // ---- merge with the other split's CTA of these rows (cluster rank
      // crank ^ 2). This pair keeps output dims [256 kp, 256 kp + 256) (the
      // TMEM block of the softmax threads with sub == kp); the other threads
      // write their O -- the peer's dims -- into the peer's staging boxes, and
      // one thread per row sends the row's (m, l).
      const int kp = (int)(crank >> 1);
      float* xml = reinterpret_cast<float*>(smem + kOffRed);            // the peer's (m, l) per row
      float* xml_out = reinterpret_cast<float*>(smem + kOffRed + 512);  // this CTA's, sent to the peer
      if (sub != kp) {
        // stage the peer's dims of O chunk by chunk (and the rows' (m, l))
        // locally; one thread ships each chunk's two boxes by bulk copy into
        // the peer's staging once the peer is ready
        if (eta == 0) {
          xml_out[2 * rho] = m_own;
          xml_out[2 * rho + 1] = ltot;
        }
        const int sender0 = 128 + 128 * (1 - kp);
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          tmem_ld32(lane_addr + o_col + 32 * c, r);
          tmem_wait_ld();
          const int d0 = 256 * sub + 128 * eta + 32 * c;
          unsigned char* row = smem + kOffStage32 + (d0 >> 5) * kBoxBytes + rho * 128;
#pragma unroll
          for (int i = 0; i < 8; ++i)
            *reinterpret_cast<uint4*>(row + (((uint32_t)i ^ sw) << 4)) =
                make_uint4(r[4 * i], r[4 * i + 1], r[4 * i + 2], r[4 * i + 3]);
          fence_proxy_async_smem();
          named_bar_sync(3, 128);
          if (threadIdx.x == sender0) {
            if (c == 0 && !mbar_wait(bar(kBarXReady), 0u, abort, wlim)) ok = false;
            const uint32_t xbar = map_to_rank(bar(kBarXData + c), xpeer);
#pragma unroll
            for (int e2 = 0; e2 < 2; ++e2) {
              const uint32_t box = sbase + kOffStage32 + (uint32_t)((8 * sub + 4 * e2 + c) * kBoxBytes);
              bulk_copy_to_cluster(map_to_rank(box, xpeer), box, kBoxBytes, xbar);
            }
            if (c == 0)
              bulk_copy_to_cluster(map_to_rank(sbase + kOffRed, xpeer), sbase + kOffRed + 512u, 64u * 8u, xbar);
          }
        }
      } else {
        const int first_keeper = 128 + 128 * kp;
        if (!mbar_wait_own(bar(kBarXData), 0u, abort, wlim)) ok = false;  // chunk 0 and the rows' (m, l)
        const float mp = xml[2 * rho], lpeer = xml[2 * rho + 1];
        const float M = fmaxf(m_own, mp);
        const float w_own = m_own == -INFINITY ? 0.0f : exp2f(m_own - M);
        const float w_p = mp == -INFINITY ? 0.0f : exp2f(mp - M);
        const float den = w_own * ltot + w_p * lpeer;
        const float dinv = den > 0.0f ? 1.0f / den : 0.0f;
        const bool keep = real_row && ok;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          const int d0 = 256 * sub + 128 * eta + 32 * c;
          uint32_t r[32];
          tmem_ld32(lane_addr + o_col + 32 * c, r);
          if (c > 0 && !mbar_wait_own(bar(kBarXData + c), 0u, abort, wlim)) ok = false;
          tmem_wait_ld();
          const unsigned char* row = smem + kOffStage32 + (d0 >> 5) * kBoxBytes + rho * 128;
          float f[32];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 v = *reinterpret_cast<const float4*>(row + (((uint32_t)i ^ sw) << 4));
            f[4 * i] = keep ? fmaf(w_p, v.x, __uint_as_float(r[4 * i]) * w_own) * dinv : 0.0f;
            f[4 * i + 1] = keep ? fmaf(w_p, v.y, __uint_as_float(r[4 * i + 1]) * w_own) * dinv : 0.0f;
            f[4 * i + 2] = keep ? fmaf(w_p, v.z, __uint_as_float(r[4 * i + 2]) * w_own) * dinv : 0.0f;
            f[4 * i + 3] = keep ? fmaf(w_p, v.w, __uint_as_float(r[4 * i + 3]) * w_own) * dinv : 0.0f;
          }
          stage_chunk(d0, f, f32_out);  // fp32: in place of the values just read
          if (!f32_out && !(c & 1)) continue;
          fence_proxy_async_smem();
          named_bar_sync(2, 128);
          if (threadIdx.x == first_keeper) {
#pragma unroll
            for (int e2 = 0; e2 < 2; ++e2) {
              if (f32_out) {
                const int j = 8 * kp + 4 * e2 + c;
                tma_store_3d(&tm_out, sbase + kOffStage32 + j * kBoxBytes, 32 * j, row0, u.b);
              } else {
                const int j = 4 * kp + 2 * e2 + (c >> 1);
                tma_store_3d(&tm_out, sbase + kOffStage16 + j * kBoxBytes, 64 * j, row0, u.b);
              }
            }
            bulk_commit();
          }
        }
        if (eta == 0 && in_range && p.lse)
          p.lse[grow] = (keep && den > 0.0f) ? (M + log2f(den)) * 0.6931471805599453f : -INFINITY;
        if (threadIdx.x == first_keeper) bulk_wait_read_all();
      }
    } else if (!merger) {
      // the final output (one split) or this split's partial
      const int kind = multi ? 0 : (f32_out ? 1 : 2);
      const float inv = !real_row ? 0.0f : ((!multi && ltot > 0.0f) ? 1.0f / ltot : 1.0f);
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(lane_addr + o_col + 32 * c, r);
        tmem_wait_ld();
        float f[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) f[i] = __uint_as_float(r[i]) * inv;
        stage_chunk(256 * sub + 128 * eta + 32 * c, f, kind != 2);
        store_chunk(c, kind);
      }
      if (grp == 0 && in_range) {
        if (multi) {
          *reinterpret_cast<float2*>(p.part_ml + ((size_t)u.split * rows_total + grow) * 2) = make_float2(m_own, ltot);
        } else if (p.lse) {
          p.lse[grow] = (real_row && ltot > 0.0f) ? (m_used + log2f(ltot)) * 0.6931471805599453f : -INFINITY;
        }
      }
      if (multi) {
        // publish: partial rows (TMA, complete) and (m, l) before the count
        if (threadIdx.x == 128) {
          bulk_wait_all();
          fence_proxy_async_global();
        }
        __threadfence();
        named_bar_sync(1, 32 * kSoftmaxWarps);
        if (threadIdx.x == 128) atomicAdd(cnt + 1, 1u);
      } else if (threadIdx.x == 128) {
        bulk_wait_read_all();
      }
    } else {
      // ---- merger
      int* s_ok = s_flag;
      if (threadIdx.x == 128) {
        bool pub = true;
        if (ld_acquire_gpu(cnt + 1) != (unsigned)(u.active - 1)) {
          const uint64_t t0 = global_timer_ns();
          while (ld_acquire_gpu(cnt + 1) != (unsigned)(u.active - 1)) {
            if (global_timer_ns() - t0 > wlim) {
              atomicExch(abort, DDT_ERR_TIMEOUT);
              pub = false;
              break;
            }
          }
        }
        if (pub) cnt[1] = 0u;
        __threadfence();
        fence_proxy_async_global();
        *s_ok = pub ? 1 : 0;
        if (pub) load_partial(u.split == 0 ? 1 : 0);
      }
      named_bar_sync(1, 32 * kSoftmaxWarps);
      const bool pub = *s_ok != 0;
      if (!pub) ok = false;
      float M = m_own;
      if (in_range && pub)
        for (int s2 = 0; s2 < u.active; ++s2)
          if (s2 != u.split) M = fmaxf(M, __ldcg(p.part_ml + ((size_t)s2 * rows_total + grow) * 2));
      const float w_own = m_own == -INFINITY ? 0.0f : exp2f(m_own - M);
      float den = w_own * ltot;
      const int nother = u.active - 1;
      int step = 0;
      for (int s2 = 0; s2 < u.active && pub; ++s2) {
        if (s2 == u.split) continue;
        float w_s = 0.0f;
        if (in_range) {
          const float2 ml = __ldcg(reinterpret_cast<const float2*>(p.part_ml) + (size_t)s2 * rows_total + grow);
          w_s = ml.x == -INFINITY ? 0.0f : exp2f(ml.x - M);
          den += w_s * ml.y;
        }
        const bool last = step == nother - 1;
        const float dinv = den > 0.0f ? 1.0f / den : 0.0f;
        const float wo = step == 0 ? w_own : 1.0f;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          if (!mbar_wait_own(bar(kBarEpi + c), (uint32_t)(step & 1), abort, wlim)) ok = false;
          const int d0 = 256 * sub + 128 * eta + 32 * c;
          uint32_t r[32];
          tmem_ld32(lane_addr + o_col + 32 * c, r);
          tmem_wait_ld();
          const unsigned char* row = smem + kOffStage32 + (d0 >> 5) * kBoxBytes + rho * 128;
          float f[32];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 v = *reinterpret_cast<const float4*>(row + (((uint32_t)i ^ sw) << 4));
            f[4 * i] = fmaf(w_s, v.x, __uint_as_float(r[4 * i]) * wo);
            f[4 * i + 1] = fmaf(w_s, v.y, __uint_as_float(r[4 * i + 1]) * wo);
            f[4 * i + 2] = fmaf(w_s, v.z, __uint_as_float(r[4 * i + 2]) * wo);
            f[4 * i + 3] = fmaf(w_s, v.w, __uint_as_float(r[4 * i + 3]) * wo);
          }
          if (last) {
            const bool keep = real_row && ok;
#pragma unroll
            for (int i = 0; i < 32; ++i) f[i] = keep ? f[i] * dinv : 0.0f;
            stage_chunk(d0, f, f32_out);  // fp32: in place of the values just read
            store_chunk(c, f32_out ? 1 : 2);
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(f[i]);
            tmem_st32(lane_addr + o_col + 32 * c, r);
          }
        }
        if (!last) {
          tmem_wait_st();
          named_bar_sync(1, 32 * kSoftmaxWarps);  // staging read by all before the next loads
          if (threadIdx.x == 128) {
            int nx = s2 + 1;
            if (nx == u.split) ++nx;
            load_partial(nx);
          }
        }
        ++step;
      }
      if (!pub) {
        // timed out waiting for the other splits: zeros
        float f[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) f[i] = 0.0f;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          stage_chunk(256 * sub + 128 * eta + 32 * c, f, f32_out);
          store_chunk(c, f32_out ? 1 : 2);
        }
      }
      if (grp == 0 && in_range && p.lse)
        p.lse[grow] = (real_row && ok && den > 0.0f) ? (M + log2f(den)) * 0.6931471805599453f : -INFINITY;
      if (threadIdx.x == 128) bulk_wait_read_all();
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

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  // looked up once per process (a function-local static initialises once,
  // whichever host thread gets here first)
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    return nullptr;
  }();
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

// [outer...][req_rows][512] row-major output-like tensor (f32 or bf16) with
// 128-byte x 64-row boxes, 128B-swizzled; rank 3 (B) or 4 (splits, B).
static bool make_out_map(CUtensorMap* m, void* base, bool f32, int rank, uint64_t req_rows, uint64_t B,
                         uint64_t splits) {
  auto fn = encode_fn();
  if (!fn) return false;
  const uint64_t es = f32 ? 4 : 2;
  cuuint64_t dims[4] = {(cuuint64_t)kDL, (cuuint64_t)req_rows, (cuuint64_t)B, (cuuint64_t)splits};
  cuuint64_t strides[3] = {(cuuint64_t)(kDL * es), (cuuint64_t)(req_rows * kDL * es),
                           (cuuint64_t)(B * req_rows * kDL * es)};
  cuuint32_t box[4] = {(cuuint32_t)(128 / es), 64, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, base,
                  dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Launch shape: how many key splits per request and whether the two splits
// of a row tile share one cluster of 4 (merged through distributed shared
// memory) or every CTA pair runs alone (merged through the workspace).
struct LaunchPlan {
  int splits;
  int csize;
};

// Pair slots: how many CTA pairs can be resident at once when the kernel runs
// in clusters of 2 (pairs4: in clusters of 4). Clusters must fit inside one
// GPC, so clusters of 4 can leave SMs of a GPC idle that pairs would use.
struct PairSlots {
  int pairs2;
  int pairs4;
};

// Makespan estimate in key tiles per pair (a tile of 256 keys is the unit):
// waves of units over the resident pairs, each unit its tiles plus a fixed
// start-up cost, plus the split merge (cheaper through distributed shared
// memory than through the workspace).
static LaunchPlan plan_launch(int B, int N, int H, int max_cache_len, PairSlots slots) {
  const int rowtiles = (N * H + 127) / 128;
  const long units1 = (long)B * rowtiles;
  const int tiles = (max_cache_len + N + kTileKeys - 1) / kTileKeys;
  const double kStart = 0.6, kMergeDsmem = 0.4, kMergeWs = 1.2;
  LaunchPlan best{1, 2};
  double best_t = 1e30;
  auto consider = [&](int s, int csize, int slots, double merge) {
    if (slots <= 0) return;
    const int per = (tiles + s - 1) / s;
    const long units = units1 * s;
    const long waves = (units + slots - 1) / slots;
    const double t = (double)waves * (per + kStart) + merge;
    if (t < best_t - 1e-9) {
      best_t = t;
      best = LaunchPlan{s, csize};
    }
  };
  for (int s = 1; s <= std::min(kMaxSplits, std::max(1, tiles)); ++s) {
    if (s == 2) consider(s, 4, slots.pairs4, kMergeDsmem);
    consider(s, 2, slots.pairs2, s > 1 ? kMergeWs : 0.0);
  }
  return best;
}

static size_t ws_header() { return 256; }

}  // namespace tc

bool tc_attn_supported(int d_l, int d_r, int in_dtype) {
  return in_dtype == DDT_BF16 && d_l == tc::kDL && d_r == tc::kDR;
}

static size_t counter_bytes(int B, int N, int H) {
  const size_t rowtiles = ((size_t)N * H + 127) / 128;
  return ((size_t)B * rowtiles * 2 * 2 * 4 + 255) / 256 * 256;
}

// Resident pairs of this kernel on the current device, looked up once per
// device (the kernel's shared-memory opt-in is set there first).
static int device_pair_slots(tc::PairSlots* out) {
  using namespace tc;
  static std::mutex mu;
  static bool done[kMaxDevices] = {};
  static PairSlots slots[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DDT_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (!done[dev]) {
    if (cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc) != cudaSuccess)
      return DDT_ERR_CUDA;
    int sms = sm_count();
    PairSlots ps{sms / 2, 0};
    for (int csize : {2, 4}) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3((unsigned)(csize * 64));
      cfg.blockDim = dim3(kThreads);
      cfg.dynamicSmemBytes = kSmemAlloc;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = (unsigned)csize;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, attn_tc_kernel, &cfg) == cudaSuccess && n > 0) {
        if (csize == 2) ps.pairs2 = n;
        else ps.pairs4 = 2 * n;
      } else {
        (void)cudaGetLastError();
      }
    }
    slots[dev] = ps;
    done[dev] = true;
  }
  *out = slots[dev];
  return DDT_OK;
}

static tc::LaunchPlan current_plan(int B, int N, int H, int max_cache_len) {
  tc::PairSlots slots{74, 64};
  (void)device_pair_slots(&slots);  // without a device: the B200's figures
  return tc::plan_launch(B, N, H, max_cache_len, slots);
}

size_t tc_attn_workspace_bytes(int B, int N, int H, int max_cache_len) {
  const int s = current_plan(B, N, H, max_cache_len).splits;
  size_t bytes = tc::ws_header();
  if (s > 1) {
    const size_t rows = (size_t)B * N * H;
    bytes += counter_bytes(B, N, H) + (size_t)s * rows * tc::kDL * 4 + (size_t)s * rows * 2 * 4;
  }
  return bytes;
}

int launch_attn_tc(const AttnParams& a, int max_cache_len, void* workspace, size_t workspace_bytes,
                   cudaStream_t stream) {
  using namespace tc;
  const int64_t kv_rows = a.kv_rows;
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
  const LaunchPlan plan = current_plan(a.B, a.N, a.H, max_cache_len);
  p.splits = plan.splits;
  p.rowtiles = (a.N * a.H + 127) / 128;
  p.out_dtype = a.out_dtype;
  p.out = a.out;
  p.lse = a.lse;
  p.dev_status = a.dev_status;
  p.kv_rows = kv_rows;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  p.abort = reinterpret_cast<int*>(ws);
  if (p.splits > 1) {
    const size_t rows = (size_t)a.B * a.N * a.H;
    const size_t cb = counter_bytes(a.B, a.N, a.H);
    p.counter = reinterpret_cast<unsigned*>(ws + ws_header());
    p.part_o = reinterpret_cast<float*>(ws + ws_header() + cb);
    p.part_ml = reinterpret_cast<float*>(ws + ws_header() + cb + (size_t)p.splits * rows * kDL * 4);
  }
  if (workspace_bytes < tc_attn_workspace_bytes(a.B, a.N, a.H, max_cache_len)) return DDT_ERR_INVALID_ARG;
  p.wait_ns = wait_limit_ns();
  // the shared-memory opt-in is a per-device function attribute: set (with
  // the pair slots) once on every device the library launches on
  {
    PairSlots slots;
    if (device_pair_slots(&slots) != DDT_OK) return DDT_ERR_CUDA;
  }
  CUtensorMap tout, tpart;
  memset(&tpart, 0, sizeof(tpart));
  if (!make_out_map(&tout, a.out, a.out_dtype == DDT_F32, 3, (uint64_t)a.N * a.H, (uint64_t)a.B, 1)) return DDT_ERR_CUDA;
  if (p.splits > 1 &&
      !make_out_map(&tpart, p.part_o, true, 4, (uint64_t)a.N * a.H, (uint64_t)a.B, (uint64_t)p.splits))
    return DDT_ERR_CUDA;
  const long long units = (long long)a.B * p.rowtiles * p.splits;
  // two key splits: both in one cluster of 4 (merged through distributed
  // shared memory); otherwise clusters of 2 (one CTA pair each)
  auto launch = [&](int csize) -> cudaError_t {
    p.csize = csize;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * units));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemAlloc;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = (unsigned)csize;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, attn_tc_kernel, tq, tkv, tout, tpart, p);
  };
  if (p.splits == 2 && plan.csize == 4) {
    if (launch(4) == cudaSuccess) return DDT_OK;
    (void)cudaGetLastError();  // clusters of 4 not schedulable here: pairs + workspace merge
  }
  return launch(2) == cudaSuccess ? DDT_OK : DDT_ERR_CUDA;
}

}  // namespace ddt
