// Target LM head folded into the accept argmax, sm_100a: the greedy token of
// every verify row, argmax_v sum_c hidden[r][c] * w_vocab[v][c], without ever
// writing the logits to memory.
//
// What it computes is fixed in ddt.h (ddt_accept_compact_lmhead): the argmax
// of the target's logits is the greedy token the walk compares against
// ("autoregressive_test_driver_kdtree_engine", section "What the Message
// Actually Says": the greedy token of a verify row is the argmax of the
// target's logits, checked exactly); the head maps the final hidden state
// (Kimi K2.6: 7168 wide; "the_validation_pivot", section "Assumptions
// Embedded in This Message") to the vocabulary.
//
// Structure: a persistent grid of CTA pairs (clusters of 2) walks the tiles
// (pass of up to 512 verify rows) x (256 vocabulary rows). The vocabulary is
// the MMA's M side (tcgen05.mma.cta_group::2, M = 256: each CTA supplies 128
// vocabulary rows of the head and holds their 128 x N fp32 accumulator in its
// tensor memory) and the verify rows are its N side (each CTA supplies half
// of them), so one head row is read from HBM once per pass however few rows
// are verified. The head and hidden tiles stream through a ring of stages by
// TMA (64 dims per stage, 128-byte swizzle); warp 0 loads, warp 1 of the
// leader CTA issues the MMAs (with two N parts, warp 6 issues the second
// part's), warps 2..5 and 7..10 reduce each finished accumulator (two warps
// per TMEM lane quarter, alternate 32-column chunks, the next chunk's TMEM
// load in flight while one is reduced): per verify row (column) the best of
// the warp's 32 vocabulary rows as a packed 64-bit key (order-preserving
// value bits << 32 | ~row: the larger key is the larger logit at the lower
// index), found by halving the columns over the lanes (5 shuffle steps per
// 32 columns, lane c ending with column c) and merged into the CTA's running
// key for that column in shared memory; the CTA's keys are published once
// per pass with a 64-bit atomic max into the same per-row keys the
// materialised-logits argmax writes, so the accept walk that follows is the
// same kernel. The accumulator is double-buffered when a pass has at most
// 256 rows, so the reduction of one tile overlaps the MMAs of the next; with
// 512 rows it fills the tensor memory and the reduction (about 15 % of a
// tile) runs between tiles.
//
// Rounding: each MMA adds 16 exact bf16 x bf16 products to the float32
// accumulator and the 64-dim stages follow one another, so a product passes
// through at most 15 + ceil(d / 16) roundings (the depth ddt.h declares).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "ddt_kernels.cuh"
#include "sm100_ptx.cuh"

namespace ddt {
namespace lmh {

using namespace sm100;

constexpr int kThreads = 352;           // warp 0 TMA, warps 1 and 6 MMA (warp 1: + TMEM), warps 2..5 and 7..10 reduction
constexpr int kABytes = 128 * 128;      // 128 head rows x 64 dims bf16 per CTA and stage
constexpr int kPassRows = 512;          // verify rows per pass over the head
constexpr int kMaxStages = 12;
constexpr int kStageBudget = 200 * 1024;

// shared memory after the stages
constexpr int kBarFull = 0;                      // [kMaxStages] leader: TMA bytes of a stage (both CTAs)
constexpr int kBarEmpty = kBarFull + kMaxStages;  // [kMaxStages] each CTA: MMAs done with a stage
constexpr int kBarAccFull = kBarEmpty + kMaxStages;  // [2] each CTA: accumulator buffer complete
constexpr int kBarAccEmpty = kBarAccFull + 2;        // [2] leader: accumulator read (8 warps x 2 CTAs)
constexpr int kNumBars = kBarAccEmpty + 2;
constexpr int kMiscBytes = 256;                  // barriers
constexpr int kSlotBytes = 16;                   // TMEM address + abort flag
constexpr int kRedBytes = kPassRows * 8;         // per-column running key of the CTA
static_assert(kNumBars * 8 <= kMiscBytes, "barrier area");

struct Params {
  int R, d, V, N;
  int nkb;        // 64-dim stages per tile
  int vtiles;     // 256-row vocabulary tiles
  int passes;     // passes of up to 512 verify rows
  int parts;      // N-parts per MMA step: 1 (pass <= 256 rows) or 2 (N = 256 each)
  int npart;      // N of one part (multiple of 16)
  int nh;         // verify rows one CTA supplies per part (npart / 2)
  int stages, stage_bytes, nbuf;
  const int32_t* n_nodes;
  unsigned long long* rowkey;
  int* abort;
  uint64_t wait_ns;
};

// Wait for this thread's TMEM loads, with the loaded registers as operands of
// the wait, so no use of them can be scheduled before it.
__device__ __forceinline__ void tmem_wait_ld_regs(uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.wait::ld.sync.aligned;"
      : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
        "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]),
        "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
        "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
      :
      : "memory");
}

__device__ __forceinline__ int ld_volatile_i32(const int* p) {
  int v;
  asm volatile("ld.volatile.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__global__ void __launch_bounds__(kThreads, 1)
    lmhead_argmax_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_h,
                         Params p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  pdl_wait();
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = (int)(blockIdx.x >> 1), npairs = (int)(gridDim.x >> 1);
  const int total = p.passes * p.vtiles;
  const uint32_t misc = sbase + (uint32_t)(p.stages * p.stage_bytes);
  auto bar = [&](int i) -> uint32_t { return misc + 8u * (uint32_t)i; };
  unsigned char* slot_area = smem + p.stages * p.stage_bytes + kMiscBytes;
  unsigned long long* s_red =
      reinterpret_cast<unsigned long long*>(smem + p.stages * p.stage_bytes + kMiscBytes + kSlotBytes);
  int* abort = p.abort;
  const uint64_t wlim = p.wait_ns;

  if (threadIdx.x == 0) {
    // with two N parts each has its own issuing thread: a stage is free, and
    // an accumulator complete, when both have committed
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(bar(kBarFull + s), 1);
      mbar_init(bar(kBarEmpty + s), (uint32_t)p.parts);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(kBarAccFull + b), (uint32_t)p.parts);
      mbar_init(bar(kBarAccEmpty + b), 16);
    }
    fence_mbar_init_cluster();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_w);
    prefetch_tmap(&tm_h);
  }
  for (int c = threadIdx.x; c < kPassRows; c += kThreads) s_red[c] = 0ull;
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(slot_area), 512);
    tmem_relinquish_pair();
  }
  // a workspace whose status word already holds an error (an earlier call
  // gave up a wait) makes the call do no work; the leader CTA reads the word
  // and both CTAs of the pair take its value
  if (leader && threadIdx.x == 0) *reinterpret_cast<volatile int*>(slot_area + 4) = ld_volatile_i32(abort);
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(slot_area);
  const bool aborted = ld_cluster_u32(map_to_rank(smem_u32(slot_area + 4), 0)) != 0u;

  if (aborted) {
    // nothing to do: straight to the teardown
  } else if (warp == 0 && lane == 0) {
    // ============================================================ TMA producer
    const uint32_t full0 = map_to_rank(bar(kBarFull), 0);
    int slot = 0;
    uint32_t phase = 0;
    bool ok = true;
    // the head streams from HBM once (evict first); the hidden rows are read
    // by every CTA for every tile (evict last)
    const uint64_t pol_w = l2_policy_evict_first(), pol_h = l2_policy_evict_last();
    for (int t = pair; t < total && ok; t += npairs) {
      const int pass = t / p.vtiles, vt = t - pass * p.vtiles;
      const int v0 = vt * 256 + 128 * (int)rank;
      const int h0 = pass * kPassRows + p.nh * (int)rank;
      for (int kb = 0; kb < p.nkb; ++kb) {
        if (!mbar_wait(bar(kBarEmpty + slot), phase ^ 1u, abort, wlim)) {
          ok = false;
          break;
        }
        if (leader) mbar_arrive_expect_tx(bar(kBarFull + slot), 2u * (uint32_t)p.stage_bytes);
        const uint32_t dst = sbase + (uint32_t)(slot * p.stage_bytes);
        const uint32_t fb = full0 + 8u * (uint32_t)slot;
        tma_load_2d_pair_hint(dst, &tm_w, 64 * kb, v0, fb, pol_w);
        for (int j = 0; j < p.parts; ++j)
          tma_load_2d_pair_hint(dst + kABytes + (uint32_t)(j * p.nh * 128), &tm_h, 64 * kb, h0 + 256 * j, fb,
                                pol_h);
        if (++slot == p.stages) {
          slot = 0;
          phase ^= 1u;
        }
      }
    }
  } else if ((warp == 1 || (warp == 6 && p.parts == 2)) && lane == 0 && leader) {
    // ============================================================ MMA issuers
    // one thread per N part (warp 6 only with two): a barrier wait in an
    // issuing thread costs the tensor pipe about two MMAs, and the other
    // thread's queued MMAs cover it; the parts' accumulators are disjoint
    const uint32_t idesc = idesc_bf16_f32(256, p.npart, false, false);
    const int j = warp == 6 ? 1 : 0;  // the N part this thread issues
    const uint32_t boff = (uint32_t)(kABytes + j * p.nh * 128);  // its hidden box in a stage
    int slot = 0;
    uint32_t phase = 0;
    bool ok = true;
    int lt = 0;
    for (int t = pair; t < total && ok; t += npairs, ++lt) {
      const int buf = lt % p.nbuf;
      if (!mbar_wait(bar(kBarAccEmpty + buf), (uint32_t)((lt / p.nbuf) & 1) ^ 1u, abort, wlim)) break;
      tc_fence_after();
      const uint32_t d = tmem + (uint32_t)((buf * p.parts + j) * 256);
      for (int kb = 0; kb < p.nkb; ++kb) {
        if (!mbar_wait(bar(kBarFull + slot), phase, abort, wlim)) {
          ok = false;
          break;
        }
        const uint32_t a0 = sbase + (uint32_t)(slot * p.stage_bytes);
        // descriptors once per stage: +32 bytes per K step is +2 in the address field
        const uint64_t da = smem_desc_sw128(a0, 16, 1024), db = smem_desc_sw128(a0 + boff, 16, 1024);
        mma_pair_ss(d, da, db, idesc, kb != 0 ? 1u : 0u);
#pragma unroll
        for (int k = 1; k < 4; ++k) mma_pair_ss(d, da + 2 * k, db + 2 * k, idesc, 1u);
        mma_commit_pair_mc(bar(kBarEmpty + slot), (uint16_t)0x3u);
        if (++slot == p.stages) {
          slot = 0;
          phase ^= 1u;
        }
      }
      if (ok) mma_commit_pair_mc(bar(kBarAccFull + buf), (uint16_t)0x3u);
    }
  } else if ((warp >= 2 && warp <= 5) || (warp >= 7 && warp <= 10)) {
    // ============================================================ reduction
    // thread = TMEM lane 32 q + lane = vocabulary row 128 rank + 32 q + lane
    // of the tile. Per 32-column chunk the warp finds, for every column
    // (verify row), the best of its 32 rows; lane c of the warp ends up with
    // column c's and merges it into the CTA's running key for that column in
    // shared memory. The loop over chunks stays rolled: the code the MMA
    // issuer runs must stay in the instruction cache next to it.
    const int q = warp & 3;                 // TMEM lane quarter (two warps each)
    const int h = warp >= 7 ? 1 : 0;        // which of the quarter's two warps: even or odd chunks
    const int rt = warp >= 7 ? (int)threadIdx.x - 224 + 128 : (int)threadIdx.x - 64;  // 0 .. 255
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * q) << 16);
    const uint32_t empty0 = map_to_rank(bar(kBarAccEmpty), 0);
    const int ncols = p.parts == 2 ? kPassRows : p.npart;
    const int nchunks = (ncols + 31) / 32;
    int cur_pass = -1;
    bool ok = true;
    // the CTA's key per column of the pass out to the rows' global keys
    auto flush = [&](int pass) {
      named_bar_sync(1, 256);
      for (int c = rt; c < ncols; c += 256) {
        const unsigned long long k = s_red[c];
        s_red[c] = 0ull;
        const int r = pass * kPassRows + c;
        if (k == 0ull || r >= p.R) continue;
        const int b = r / p.N, i = r - b * p.N;
        if (i < __ldg(p.n_nodes + b)) atomicMax(p.rowkey + r, k);
      }
      named_bar_sync(1, 256);
    };
    named_bar_sync(1, 256);  // the 8 warps start together (s_red was zeroed before the set-up barrier)
    int lt = 0;
    for (int t = pair; t < total; t += npairs, ++lt) {
      const int pass = t / p.vtiles, vt = t - pass * p.vtiles;
      if (pass != cur_pass) {
        if (cur_pass >= 0) flush(cur_pass);
        cur_pass = pass;
      }
      const int buf = lt % p.nbuf;
      if (ok && !mbar_wait(bar(kBarAccFull + buf), (uint32_t)((lt / p.nbuf) & 1), abort, wlim)) ok = false;
      tc_fence_after();
      const int vrow = vt * 256 + 128 * (int)rank + 32 * q + lane;  // this thread's vocabulary row
      const bool valid = ok && vrow < p.V;
      const uint32_t col0 = (uint32_t)(buf * p.parts * 256);
      // per column, the best (value, lowest row) over the warp's 32 rows as
      // packed keys (order-preserving value << 32 | ~row), by halving: at
      // width h a lane keeps the upper h columns of its 2h if its h bit is
      // set, the lower ones otherwise, and takes the larger of its key and
      // its partner's (lane ^ h) for each; after h = 16 .. 1 lane l holds
      // column l of the chunk
      auto reduce = [&](const uint32_t (&r)[32], int m) {
        unsigned long long k[32];
#pragma unroll
        for (int i = 0; i < 32; ++i)
          k[i] = valid ? ((unsigned long long)float_order_key(__uint_as_float(r[i])) << 32) |
                             (unsigned long long)(~(uint32_t)vrow)
                       : 0ull;
#pragma unroll
        for (int h = 16; h >= 1; h >>= 1) {
          const bool up = (lane & h) != 0;
#pragma unroll
          for (int i = 0; i < h; ++i) {
            const unsigned long long keep = up ? k[i + h] : k[i];
            const unsigned long long send = up ? k[i] : k[i + h];
            const unsigned long long got = __shfl_xor_sync(DDT_FULL_MASK, send, h);
            k[i] = got > keep ? got : keep;
          }
        }
        if (k[0] != 0ull) atomicMax(s_red + 32 * m + lane, k[0]);
      };
      // after this warp's last chunk's load its columns of the accumulator
      // are in registers: once all eight warps of both CTAs have arrived the
      // buffer is free for the next tile's MMAs
      auto release = [&]() {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (leader) mbar_arrive_local(bar(kBarAccEmpty + buf));
          else mbar_arrive_cluster(empty0 + 8u * (uint32_t)buf);
        }
      };
      // this warp's chunks h, h + 2, ...; two register buffers: the next
      // one loads while this one is reduced
      const int cnt = nchunks > h ? (nchunks - h + 1) / 2 : 0;
      auto col = [&](int j) { return lane_addr + col0 + 32u * (uint32_t)(h + 2 * j); };
      uint32_t ra[32], rb[32];
      if (cnt == 0) release();  // nothing to read in this buffer
      else tmem_ld32(col(0), ra);
#pragma unroll 1
      for (int j = 0; j < cnt; j += 2) {
        tmem_wait_ld_regs(ra);
        if (j + 1 < cnt) tmem_ld32(col(j + 1), rb);
        if (j + 1 == cnt) release();
        reduce(ra, h + 2 * j);
        if (j + 1 < cnt) {
          tmem_wait_ld_regs(rb);
          if (j + 2 < cnt) tmem_ld32(col(j + 2), ra);
          if (j + 2 == cnt) release();
          reduce(rb, h + 2 * (j + 1));
        }
      }
    }
    if (cur_pass >= 0) flush(cur_pass);
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

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// [rows][d] bf16, row-major: boxes of 64 dims x box_rows rows, 128-byte swizzle
static bool make_map(CUtensorMap* m, const void* base, uint64_t d, uint64_t rows, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static int smem_bytes(const Params& p) {
  return p.stages * p.stage_bytes + kMiscBytes + kSlotBytes + kRedBytes + 1024;
}

// CTA pairs of this kernel that can be resident at once on the current
// device, looked up once per device (with the shared-memory opt-in set).
static int device_pairs(int smem) {
  static std::mutex mu;
  static int pairs[kMaxDevices] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
  std::lock_guard<std::mutex> lock(mu);
  if (cudaFuncSetAttribute(lmhead_argmax_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kStageBudget + kMiscBytes + kSlotBytes + kRedBytes + 1024) != cudaSuccess)
    return -1;
  if (pairs[dev] == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * 64);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = (size_t)smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, lmhead_argmax_kernel, &cfg) != cudaSuccess || n <= 0) {
      (void)cudaGetLastError();
      n = sm_count() / 2;
    }
    pairs[dev] = n;
  }
  return pairs[dev];
}

}  // namespace lmh

bool lmhead_supported(int d_model, int V, const void* hidden, const void* w_vocab) {
  return d_model >= 8 && d_model % 8 == 0 && V >= 1 && (reinterpret_cast<uintptr_t>(hidden) % 16) == 0 &&
         (reinterpret_cast<uintptr_t>(w_vocab) % 16) == 0;
}

int launch_lmhead_argmax(const void* hidden, const void* w_vocab, int d_model, int V, int B, int N,
                         const int32_t* n_nodes, void* workspace, cudaStream_t stream) {
  using namespace lmh;
  Params p{};
  p.R = B * N;
  p.d = d_model;
  p.V = V;
  p.N = N;
  p.nkb = (d_model + 63) / 64;
  p.vtiles = (V + 255) / 256;
  if (p.R <= 256) {
    p.parts = 1;
    p.npart = std::max(16, (p.R + 15) / 16 * 16);
    p.passes = 1;
    p.nbuf = 2;
  } else {
    p.parts = 2;
    p.npart = 256;
    p.passes = (p.R + kPassRows - 1) / kPassRows;
    p.nbuf = 1;
  }
  p.nh = p.npart / 2;
  p.stage_bytes = kABytes + p.parts * p.nh * 128;
  p.stages = std::min(kMaxStages, kStageBudget / p.stage_bytes);
  p.n_nodes = n_nodes;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  p.abort = reinterpret_cast<int*>(ws);
  p.rowkey = reinterpret_cast<unsigned long long*>(ws + 256);
  p.wait_ns = wait_limit_ns();
  CUtensorMap tw, th;
  if (!make_map(&tw, w_vocab, (uint64_t)d_model, (uint64_t)V, 128) ||
      !make_map(&th, hidden, (uint64_t)d_model, (uint64_t)p.R, (uint32_t)p.nh))
    return DDT_ERR_CUDA;
  const int smem = smem_bytes(p);
  const int slots = device_pairs(smem);
  if (slots <= 0) return DDT_ERR_CUDA;
  const long long tiles = (long long)p.passes * p.vtiles;
  const int pairs = (int)std::max<long long>(1, std::min<long long>(slots, tiles));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * pairs));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, lmhead_argmax_kernel, tw, th, p) == cudaSuccess ? DDT_OK : DDT_ERR_CUDA;
}

}  // namespace ddt
