/*
 * ddt.h -- C ABI of libddt.so: one DDTree speculative-decoding tree-verify
 * step on an NVIDIA B200 (sm_100a).
 *
 * The step has three calls, issued in this order on one CUDA stream (a
 * fourth, ddt_drafter_topk, can produce the build's inputs from the
 * drafter's logits):
 *
 *   ddt_build_tree      best-first draft tree from the drafter's per-depth
 *                       top-k log-probs ("autoregressive_test_driver_kdtree_
 *                       engine", section "The Broader Context": GPU best-first
 *                       tree builder replacing a per-request CPU heapq;
 *                       "ddtree_speculative_decode_test_capstone", section
 *                       "What the Test Validated": the drafter contract);
 *   ddt_verify_attn     MLA-absorb attention of every tree node's heads over the
 *                       request's latent KV cache plus its visible tree
 *                       ancestors (first page, "The Broader Context":
 *                       tree-verify MLA-absorb attention with visibility
 *                       masking);
 *   ddt_accept_compact  greedy accept walk over the target's argmax and
 *                       compaction of the accepted nodes' latent KV rows into
 *                       the contiguous cache (first page, "The Broader
 *                       Context": greedy tree-accept kernel, KV cache with
 *                       post-verify compaction).
 *
 * Common conventions
 *   - Every pointer argument is DEVICE memory owned by the caller, except where
 *     a comment says "host". The library allocates no device memory: scratch
 *     comes from a caller-provided workspace whose size a *_workspace_size()
 *     query returns.
 *   - Calls are asynchronous and stream-ordered on `stream` (0 = legacy default
 *     stream); none synchronises the host. Calls on different streams with
 *     disjoint buffers may run concurrently.
 *   - The return value is a ddt_status. Host-side argument checks (null
 *     pointers, sizes, unsupported shapes or dtypes) are synchronous and
 *     launch nothing. A failed launch returns DDT_ERR_CUDA.
 *   - Device-side preconditions (bad drafter log-probs, cache capacity, a
 *     request's rows inside the pool) never trap: the kernel writes a ddt_status value to dev_status[b] (when
 *     dev_status is non-null, else the problem is only visible through the
 *     padded outputs) and skips that request as documented per call.
 *   - Shapes: B requests, D drafter depth, K top-k, N verify rows per request
 *     INCLUDING the root (N - 1 drafted nodes; block_size = budget + 1 on the
 *     capstone page), H heads, d_l latent dim, d_r RoPE dim, d_qk = d_l + d_r,
 *     V vocab, W = ceil(N / 32) mask words. Arrays are row-major, innermost
 *     index last.
 *   - Limits: 1 <= N <= 1024, 1 <= K <= 32, 1 <= D <= 64, B >= 1, and the
 *     tree's tie-break key (ceil(log2 K) bits per level, min(D, N - 1) levels)
 *     must fit 64 bits, else DDT_ERR_UNSUPPORTED.
 */
#ifndef DDT_H_
#define DDT_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define DDT_API __attribute__((visibility("default")))
#else
#define DDT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DDT_OK = 0,
  DDT_ERR_INVALID_ARG = 1, /* null pointer, size out of range, bad workspace */
  DDT_ERR_UNSUPPORTED = 2, /* valid but not implemented (shape / dtype combo) */
  DDT_ERR_CAPACITY = 3,    /* device: cache_len + n_nodes > cache_cap         */
  DDT_ERR_INPUT = 4,       /* device: drafter log-probs violate preconditions */
  DDT_ERR_CUDA = 5,        /* a CUDA launch or driver call failed             */
  DDT_ERR_TIMEOUT = 6,     /* device: a bounded intra-kernel wait gave up     */
  DDT_ERR_BOUNDS = 7       /* device: a request's rows fall outside the pool  */
} ddt_status;

typedef enum { DDT_F32 = 0, DDT_BF16 = 1 } ddt_dtype;

/* Human-readable name of a status code (static string, never null). */
DDT_API const char* ddt_status_string(int status);

/* Library version, major * 10000 + minor * 100 + patch. */
DDT_API int ddt_version(void);

/*
 * ddt_set_wait_limit_ns -- wall-clock limit of every bounded wait inside the
 * library's kernels (a barrier a pipeline stage waits on, a counter another
 * CTA must advance). A wait that runs past it gives up: the kernel stores
 * DDT_ERR_TIMEOUT in the call's workspace status word and returns instead of
 * spinning. Process-wide; read when a kernel is launched, so it applies to
 * calls issued after this one. 0 restores the default (2 s); values below
 * 1 ms are raised to 1 ms. Returns the previous limit. Host only, thread-safe.
 */
DDT_API uint64_t ddt_set_wait_limit_ns(uint64_t ns);

/*
 * ddt_drafter_topk -- the drafter's per-depth proposals from its logits: for
 * every row (one request's depth), the log-softmax over the vocabulary and
 * the K best tokens, best first. Its outputs are ddt_build_tree's logp / tok
 * inputs (rows = B * D, row-major [B][D]).
 *
 * Passage: capstone page, "The Oracle Drafter" (the drafter hands the tree
 * builder per-depth log-probabilities and token ids of its candidates, sorted
 * best first); first page, "The Broader Context" (the draft tree is built
 * from the drafter's per-depth top-k). The pages fix no formula: the plainest
 * reading is used.
 *
 * Definition: tok[r][k] = the index of the k-th largest logits[r][v] (equal
 *   values: the lower index first; bf16 widened exactly to float32);
 *   logp[r][k] = logits[r][tok[r][k]] - logsumexp_v(logits[r][v]), float32
 *   arithmetic (the log-sum-exp is a float32 running sum of 2^(x log2 e - max)).
 * Inputs (device): logits [R][V] logits_dtype (F32 or BF16), finite.
 * Outputs (device): logp [R][K] float32, tok [R][K] int32; dev_status [R]
 *   (nullable): DDT_OK, or DDT_ERR_INPUT for a row holding a non-finite
 *   logit (that row's tok = -1, logp = -inf).
 * Sizes: R >= 1, V >= 1, 1 <= K <= min(V, 32); R < 2^28 and V <= 2^30
 *   (DDT_ERR_UNSUPPORTED beyond).
 * A row is split over a cluster of min(8, ceil(V / 16384), SMs / R) CTAs
 *   (at least one; one CTA per row where such a cluster cannot be
 *   scheduled), so the launch is one wave; no workspace. Errors:
 *   DDT_ERR_INVALID_ARG (nulls, sizes, dtype), DDT_ERR_UNSUPPORTED (sizes
 *   above), DDT_ERR_CUDA (launch).
 */
DDT_API int ddt_drafter_topk(const void* logits, int logits_dtype, int V, int R, int K, float* logp,
                             int32_t* tok, int32_t* dev_status, cudaStream_t stream);

/*
 * ddt_build_tree -- best-first draft tree for every request.
 *
 * Passage: capstone page, "What the Test Validated" (a drafter returns, per
 * depth up to a limit, log-probs and token ids of its top-k candidates, sorted
 * so the tree builder's best-first search takes the best first) and first
 * page, "The Broader Context" (GPU best-first builder replacing a heapq).
 *
 * Definition (readings the pages leave open are fixed here):
 *   A rank path r = (r_1..r_d), 1 <= d <= D, scores the float32 sum
 *   s = (((0 + logp[b][0][r_1]) + logp[b][1][r_2]) + ...) added left to right
 *   in round-to-nearest (no fused or reassociated adds). Paths are ordered by
 *   (s descending, d ascending, (r_1..r_d) lexicographically ascending); the
 *   tree holds the first min(N - 1, sum_d K^d) of them. Node 0 is the root
 *   (previous step's bonus token); node i >= 1 is the i-th path in order, so
 *   parent[i] < i. tok = tok[b][d-1][r_d], depth = d, pos = cache_len[b] + d,
 *   score = s. mask row i has bit j (word j >> 5, bit j & 31) set iff node j is
 *   node i or one of its ancestors.
 *
 * Inputs (device):
 *   logp      [B][D][K] float32, per depth non-increasing in k, finite, <= 0.
 *   tok       [B][D][K] int32 candidate token ids.
 *   root_tok  [B] int32, cache_len [B] int32 (committed rows before the step).
 * Outputs (device, fully written for all N rows):
 *   node_tok, parent, depth, pos [B][N] int32; score [B][N] float32;
 *   mask [B][N][W] uint32; n_nodes [B] int32.
 *   Pad rows i >= n_nodes[b]: node_tok/parent/depth/pos = -1, score = -inf,
 *   mask = 0.
 *   dev_status [B] int32 (nullable): DDT_OK, or DDT_ERR_INPUT when logp[b]
 *   breaks its precondition -- that request then gets n_nodes = 0 and every
 *   row padded.
 * One warp per request (a best-first search; for 128 < N <= 256 with D <= 16
 * and K <= 16 and rank tuples wider than 25 bits, one CTA of 512 threads per
 * request that selects the best N - 1 paths depth by depth with radix
 * selects, the same nodes in the same order); no workspace.
 */
DDT_API int ddt_build_tree(const float* logp, const int32_t* tok, const int32_t* root_tok,
                   const int32_t* cache_len, int B, int D, int K, int N,
                   int32_t* node_tok, int32_t* parent, int32_t* depth, int32_t* pos,
                   float* score, uint32_t* mask, int32_t* n_nodes, int32_t* dev_status,
                   cudaStream_t stream);

/*
 * ddt_verify_attn -- MLA-absorb tree-verify attention.
 *
 * Passage: first page, "The Broader Context" (tree-verify MLA-absorb
 * attention kernel with visibility masking) and capstone page, "Context and
 * Motivation" (the target verifies the drafted tree in one batched forward).
 *
 * Definition: each pool row is [c (d_l latent) ; k_pe (d_r RoPE key)]; the key
 * is the whole row, the value its first d_l entries (absorbed MLA: one latent
 * row serves every head). For request b, node i < n_nodes[b], head h:
 *   visible keys j: every committed row j in [0, cache_len[b]) and tree row
 *                   cache_len[b] + t for each node t < n_nodes[b] whose bit is
 *                   set in mask[b][i];
 *   s_j = scale * dot(q[b][i][h][:], kv[cache_off[b] + j][:])   (d_qk terms)
 *   out[b][i][h][:] = sum_j softmax(s)_j * kv[cache_off[b] + j][0:d_l]
 *   lse[b][i][h]    = ln sum_j exp(s_j)
 * Pad rows (i >= n_nodes[b]): out = 0, lse = -inf.
 *
 * Inputs (device):
 *   q         [B][N][H][d_qk] in_dtype; q_pe and k_pe already RoPE-rotated.
 *   kv        pool [kv_rows][d_qk] in_dtype. Request b's rows start at
 *             cache_off[b]: cache_len[b] committed rows, then the N tree rows
 *             in node order (tree row t = node t's latent row).
 *   cache_off [B] int64, cache_len [B] int32, mask [B][N][W] uint32,
 *             n_nodes [B] int32 (as written by ddt_build_tree).
 *   max_cache_len (host): an upper bound on every cache_len[b]; it sizes the
 *             launch and the workspace. kv_rows (host): rows in the pool.
 * Outputs (device): out [B][N][H][d_l] out_dtype; lse [B][N][H] float32
 *   (nullable); dev_status [B] int32 (nullable): DDT_OK, or DDT_ERR_BOUNDS
 *   when cache_off[b] + cache_len[b] + n_nodes[b] > kv_rows, a value is
 *   negative, or n_nodes[b] > N -- all that request's rows are then written
 *   as pad rows (the bf16 kernel may already have read committed rows
 *   through TMA, which returns zeros outside the pool; the f32 kernel reads
 *   nothing) -- or DDT_ERR_TIMEOUT when the workspace's status word already
 *   held a timeout (bf16 kernel).
 * Launch order: the bf16 kernel is launched as a programmatic dependent and
 *   may start while the kernel before it on the stream still runs, if that
 *   kernel allows it (of this library's kernels, the tree build does: the
 *   verify attention then computes over the committed cache while the tree
 *   is built). It reads q, kv, cache_off and cache_len at once, and waits
 *   for the preceding kernel before it reads mask or n_nodes. So q, kv,
 *   cache_off and cache_len must not be written by the kernel issued just
 *   before this call; the library's kernels that write the pool or
 *   cache_len (the accept's walk and compaction) never let a dependent start
 *   early, and kernels that are not programmatic-launch aware never do.
 * Supported: in_dtype F32 (CUDA-core kernel, any d_l, d_r with d_qk <= 1024)
 *   and BF16 with (d_l, d_r) = (512, 64) (tensor-core kernel); out_dtype F32
 *   or BF16. Accumulation is float32 throughout. The bf16 kernel rounds the
 *   softmax probabilities to bf16 before the P.V product.
 * workspace: at least ddt_verify_attn_workspace_size(...) bytes of device
 *   memory, 256-byte aligned (may be null when that size is 0). Its first 256
 *   bytes are a device status word that must be zero before the first call
 *   (zero the buffer once after allocating it). Every wait inside the bf16
 *   kernel is bounded (ddt_set_wait_limit_ns, default 2 s); if one expires the
 *   kernel stores DDT_ERR_TIMEOUT there, writes zeros for the rows it could
 *   not finish and returns, and later calls with that workspace give up their
 *   waits at once until the caller zeroes it again. When the launch splits
 *   the keys (the size above 256), the next bytes are per-row-tile arrival
 *   counters that must also start at zero; each call leaves them at zero
 *   (except after a timeout: zero the whole workspace then). The rest holds
 *   per-split partial results; its contents do not matter. Calls that share
 *   a workspace must not overlap in time.
 * Pool bounds: both kernels check, per request, that its rows lie in the
 *   pool (see dev_status) before reading any. cache_len[b] <= max_cache_len
 *   is a precondition of speed only: the launch is sized for max_cache_len.
 * Errors: DDT_ERR_INVALID_ARG (nulls, sizes, workspace too small or
 *   misaligned, kv / q not 16-byte aligned for bf16), DDT_ERR_UNSUPPORTED.
 */
DDT_API size_t ddt_verify_attn_workspace_size(int B, int N, int H, int d_latent, int d_rope,
                                      int max_cache_len, int in_dtype);

DDT_API int ddt_verify_attn(const void* q, const void* kv, int64_t kv_rows, const int64_t* cache_off,
                    const int32_t* cache_len, const uint32_t* mask, const int32_t* n_nodes,
                    int B, int N, int H, int d_latent, int d_rope, float scale,
                    int max_cache_len, int in_dtype, int out_dtype, void* out, float* lse,
                    int32_t* dev_status, void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * ddt_accept_compact -- greedy accept walk, then latent-KV compaction.
 *
 * Passage: first page, "The Broader Context" (greedy tree-accept kernel; KV
 * cache with post-verify compaction); capstone page, "What the Test
 * Validated" (the target's prediction at the last accepted node is the bonus
 * token; budget = block size - 1 leaves room for it).
 *
 * Definition: am[b][i] = the lowest index of the largest logit of row i
 * (logits compared exactly; bf16 widened to float32). Walk: cur = 0; while some
 * child c of cur has node_tok[b][c] == am[b][cur], move to the lowest such c.
 * The path (root first) has a + 1 nodes; acc_len[b] = a. Committed tokens:
 * out_tok[b][0..a] = the a accepted nodes' tokens, then bonus[b] =
 * am[b][path[a]]. Compaction, on every layer l:
 *   kv[l*layer_stride_rows + cache_off[b] + cache_len[b] + j]
 *       <- kv[l*layer_stride_rows + cache_off[b] + cache_len[b] + path[j]],
 *   j = 0..a, every source row read before any is written; then
 *   cache_len[b] += a + 1.
 *
 * Inputs (device): logits [B][N][V] logits_dtype, finite; node_tok, parent
 *   [B][N] int32 and n_nodes [B] (from ddt_build_tree); kv pool of kv_rows
 *   (host value: every layer's rows) rows of row_elems elements of kv_dtype
 *   (row_elems * element size a multiple of 4 bytes); cache_off [B] int64;
 *   cache_cap [B] int32 (rows owned by b).
 * In/out: cache_len [B] int32 (advanced by a + 1).
 * Outputs (device): am [B][N] int32 (nullable; -1 on pad rows), acc_len [B],
 *   acc_nodes [B][N] (path, -1 padded), out_tok [B][N] (-1 padded), bonus [B].
 *   dev_status [B] (nullable): DDT_OK; DDT_ERR_INPUT when n_nodes[b] > N;
 *   DDT_ERR_BOUNDS when a row the compaction may touch,
 *   l*layer_stride_rows + cache_off[b] + [cache_len[b], cache_len[b] +
 *   n_nodes[b]) for some layer l, lies outside [0, kv_rows);
 *   DDT_ERR_CAPACITY when cache_len[b] + n_nodes[b] > cache_cap[b]. Each of
 *   these skips the request: acc_len 0, bonus -1, nothing copied, cache_len
 *   unchanged. Requests with n_nodes[b] == 0 are skipped the same way with
 *   DDT_OK.
 * workspace: ddt_accept_compact_workspace_size(B, N, V) bytes, 256-byte
 *   aligned: a 256-byte header (the status word at byte 0, the argmax's
 *   seven work counters at bytes 32, 64, ..., 224), then one 8-byte running
 *   argmax key per row (B * N,
 *   rounded up to 256 bytes). All of it must be zero before the first call --
 *   zero the buffer once after allocating it; every call that returns DDT_OK
 *   leaves it at zero again (after a call that returned an error, zero it
 *   again before the next). The argmax kernel waits (bounded, see
 *   ddt_set_wait_limit_ns) for its own bulk copies; if a wait gives up, the
 *   status word holds DDT_ERR_TIMEOUT, every request reports
 *   DDT_ERR_TIMEOUT and accepts nothing, and later calls with that
 *   workspace do the same until the caller zeroes it. Calls that share a
 *   workspace must not overlap on the GPU.
 * Precondition the library cannot check: the layers and requests own
 *   disjoint rows.
 * Runs as two kernels (three with several layers): the logits stream once,
 *   warps taking chunks of 2048-entry row slices from the work counters
 *   (few rows: brought into a 3-deep shared-memory ring by 1-D bulk copies;
 *   otherwise 16-byte loads), row maxima published by 64-bit atomic max; then
 *   one CTA per request finds each node's accepted child, walks the path and
 *   (one layer) compacts the rows; with several layers a third kernel moves
 *   the rows, spread over (request, layer group) CTAs.
 * Launch order: the argmax kernel is a programmatic dependent and reads only
 *   logits and the workspace, every row of the logits (pad rows too), so it
 *   may start while the kernel before it in the stream still runs (this
 *   library's tree build and verify attention let dependents start early);
 *   it waits for that kernel before it ends, and the walk and compaction run
 *   after it. So the logits must not be written by a kernel just before the
 *   call that lets its dependents start early; kernels that are not
 *   programmatic-launch aware never do.
 */
DDT_API size_t ddt_accept_compact_workspace_size(int B, int N, int V);

DDT_API int ddt_accept_compact(const void* logits, int logits_dtype, int V, const int32_t* node_tok,
                       const int32_t* parent, const int32_t* n_nodes, int B, int N, void* kv,
                       int64_t kv_rows, int kv_dtype, int row_elems, int n_layers, int64_t layer_stride_rows,
                       const int64_t* cache_off, int32_t* cache_len, const int32_t* cache_cap,
                       int32_t* am, int32_t* acc_len, int32_t* acc_nodes, int32_t* out_tok,
                       int32_t* bonus, int32_t* dev_status, void* workspace,
                       size_t workspace_bytes, cudaStream_t stream);

/*
 * ddt_accept_compact_lmhead -- ddt_accept_compact with the target's LM head
 * folded into the argmax: the verify rows' greedy tokens come straight from
 * their final hidden states and the head's weights, and the logits are never
 * written to memory.
 *
 * Passage: first page, "What the Message Actually Says" (the greedy token of
 * a verify row is the argmax of the target's logits, checked exactly);
 * "the_validation_pivot", "Assumptions Embedded in This Message" (the head
 * maps the final hidden state, 7168 wide on Kimi K2.6, to the vocabulary).
 *
 * Definition: am[b][i] = the lowest v among those with the largest
 *   z[v] = sum_c hidden[b][i][c] * w_vocab[v][c]; then the walk, outputs and
 *   compaction of ddt_accept_compact. z is evaluated in float32: every
 *   bf16 x bf16 product is exact, and a product passes through at most
 *   15 + ceil(d_model / 16) float32 roundings (16-product tensor-core steps
 *   added in sequence). Where several tokens lie within that rounding of
 *   the maximum, any of them may be picked.
 * Inputs (device): hidden [B][N][d_model] bf16 (rows i >= n_nodes[b] are
 *   read but ignored), w_vocab [V][d_model] bf16 (one row per token); both
 *   16-byte aligned, d_model a multiple of 8. The other arguments, the
 *   outputs and the device statuses are ddt_accept_compact's, with one more
 *   status: DDT_ERR_TIMEOUT in dev_status[b] (and in the workspace's first
 *   word) when a bounded wait inside the head kernel gave up -- nothing is
 *   accepted then; zero the workspace before reusing it.
 * workspace: ddt_accept_compact_workspace_size(B, N, V) bytes, zeroed once
 *   after allocation, left zeroed by every call that does not time out.
 * Runs as two kernels: a persistent 2-CTA tcgen05 GEMM with the vocabulary
 *   as M (256 head rows per CTA pair, streamed by TMA, read once per pass of
 *   up to 512 verify rows) and the verify rows as N, whose epilogue reduces
 *   every tensor-memory tile to per-row (max, lowest index) keys; then the
 *   walk and compaction kernel of ddt_accept_compact.
 * Errors: ddt_accept_compact's, and DDT_ERR_UNSUPPORTED for d_model not a
 *   multiple of 8 or misaligned hidden / w_vocab.
 */
DDT_API int ddt_accept_compact_lmhead(const void* hidden, const void* w_vocab, int d_model, int V,
                                      const int32_t* node_tok, const int32_t* parent, const int32_t* n_nodes,
                                      int B, int N, void* kv, int64_t kv_rows, int kv_dtype, int row_elems,
                                      int n_layers, int64_t layer_stride_rows, const int64_t* cache_off,
                                      int32_t* cache_len, const int32_t* cache_cap, int32_t* am, int32_t* acc_len,
                                      int32_t* acc_nodes, int32_t* out_tok, int32_t* bonus, int32_t* dev_status,
                                      void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * ddt_accept_compact_noalloc -- ddt_accept_compact without a workspace.
 *
 * No counterpart in the paper: this is a convenience of this library. Some
 * callers cannot allocate device memory at the point where they verify a
 * tree -- for example code that is only handed fixed, pre-reserved buffers by
 * the host application, or a latency-critical decode loop that must not call
 * cudaMalloc (which can synchronise the device). This entry point takes the
 * same arguments as ddt_accept_compact minus the workspace and allocates
 * nothing: its scratch (status word, work counters and per-row argmax keys) lives in one
 * fixed 4 MiB array inside the library, which every GPU
 * that loads the library keeps until the process exits.
 *
 * Limit: ddt_accept_compact_workspace_size(B, N, V) must be at most 4 MiB
 *   (e.g. B 64 x N 256 needs 0.13 MiB, B 512 x N 1024 needs 4.0 MiB + 256 B
 *   and is rejected); larger calls return
 *   DDT_ERR_UNSUPPORTED without launching anything.
 * Set-up: the first call on each device looks up the array's device address
 *   (with that device current); make that first call before any stream
 *   capture. The address is kept for the life of the process, so do not use
 *   the library across cudaDeviceReset.
 * Sharing: every call on every stream uses the same array, which keeps what
 *   the last call left in it. Each call first clears the counters it needs on
 *   its own stream; calls that overlap on the GPU race on the array and give
 *   wrong results, so serialise them (one stream, or events).
 * Everything else -- definition, layouts, outputs, device status -- is as for
 * ddt_accept_compact.
 */
DDT_API int ddt_accept_compact_noalloc(const void* logits, int logits_dtype, int V, const int32_t* node_tok,
                                       const int32_t* parent, const int32_t* n_nodes, int B, int N, void* kv,
                                       int64_t kv_rows, int kv_dtype, int row_elems, int n_layers, int64_t layer_stride_rows,
                                       const int64_t* cache_off, int32_t* cache_len, const int32_t* cache_cap,
                                       int32_t* am, int32_t* acc_len, int32_t* acc_nodes, int32_t* out_tok,
                                       int32_t* bonus, int32_t* dev_status, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* DDT_H_ */
