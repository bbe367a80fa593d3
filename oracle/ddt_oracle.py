"""CPU oracle for the DDTree tree-verify step (test infrastructure).

This module is the plain, slow, obviously-correct statement of what one
tree-verify step computes. It exists only to check the CUDA library: tests,
the smoke check and the benchmark's CPU-baseline leg may call it; the product
path never does. It shares no code with the CUDA side; both are fed by the
seeded generator in ``ddtree_speculative_decode_b200.synth``.

Sources. The pages ("autoregressive_test_driver_kdtree_engine", "ddtree_
speculative_decode_test_capstone", "the_validation_pivot") describe three
kernels -- a best-first tree builder fed by per-depth top-k log-probs, an
MLA-absorb tree-verify attention with visibility masking, and a greedy
tree-accept followed by KV-cache compaction -- but print no formulas. Where
they are silent this file takes the plainest reading; every such reading is
marked READING below.

Conventions (arrays are numpy):
  B requests, D drafter depth, K top-k, N verify rows per request including
  the root (N - 1 drafted nodes), H heads, d_l latent dim, d_r rope dim,
  V vocab, W = ceil(N / 32) mask words.

Two steps around the path are here as well: the drafter's per-depth
proposals (log-softmax + top-k over the vocabulary) feeding the build, and the
target's LM head folded into the accept argmax (logits never stored).

Parity status: every function here is pinned by tests in tests/test_oracle_*.
"""
from __future__ import annotations

import heapq
import math

import numpy as np

OK = 0
ERR_INPUT = 4
ERR_CAPACITY = 3

# ---------------------------------------------------------------------------
# a1: best-first tree build
# ---------------------------------------------------------------------------


def _drafter_ok(logp_b: np.ndarray) -> bool:
    """Precondition on one request's drafter output: finite log-probs, <= 0,
    non-increasing along the top-k axis (the sorted candidates the builder is
    handed; capstone page, "What the Test Validated")."""
    if not np.all(np.isfinite(logp_b)):
        return False
    if np.any(logp_b > 0):
        return False
    if logp_b.shape[1] > 1 and np.any(logp_b[:, 1:] > logp_b[:, :-1]):
        return False
    return True


def build_tree(logp, tok, root_tok, cache_len, N):
    """Best-first draft-tree build for every request.

    Capstone page, "What the Test Validated": the builder runs a best-first
    search over the drafter's per-depth candidates (sorted, best first) and the
    first page's "Broader Context" says it replaced a per-request CPU heapq.
    READING (scores): a rank path r = (r_1..r_d) scores the float32 sum
    s = (((0 + logp[0][r_1]) + logp[1][r_2]) + ...) evaluated left to right.
    READING (order): paths are ranked by (score descending, depth ascending,
    rank tuple lexicographically ascending); the tree is the first
    min(N - 1, sum_d K^d) paths in that order. With log-probs <= 0 and sorted,
    each path's prefix and left sibling rank before it, so a heap that starts
    from (rank 0 at depth 1) and, on each pop, pushes the first child and the
    next sibling pops paths in exactly that order; this function runs that heap.
    READING (budget): N counts verify rows including the root, as block_size 8
    = root + budget 7 on the capstone page.

    Node 0 is the root (token root_tok, depth 0, parent -1, score 0); node i >= 1
    is the i-th popped path. pos = cache_len + depth. mask row i has bit j set
    (word j >> 5, bit j & 31) iff node j is node i or one of its ancestors.
    Pad rows (i >= n_nodes): token/parent/depth/pos -1, score -inf, mask 0.
    A request whose drafter output breaks the precondition gets n_nodes = 0,
    all rows padded, status ERR_INPUT.
    """
    logp = np.asarray(logp, np.float32)
    tok = np.asarray(tok, np.int32)
    B, D, K = logp.shape
    W = (N + 31) // 32
    out = {
        "node_tok": np.full((B, N), -1, np.int32),
        "parent": np.full((B, N), -1, np.int32),
        "depth": np.full((B, N), -1, np.int32),
        "pos": np.full((B, N), -1, np.int32),
        "score": np.full((B, N), -np.inf, np.float32),
        "mask": np.zeros((B, N, W), np.uint32),
        "n_nodes": np.zeros(B, np.int32),
        "status": np.zeros(B, np.int32),
    }
    for b in range(B):
        if not _drafter_ok(logp[b]):
            out["status"][b] = ERR_INPUT
            continue
        nodes = _best_first(logp[b], N - 1)
        # root
        out["node_tok"][b, 0] = root_tok[b]
        out["parent"][b, 0] = -1
        out["depth"][b, 0] = 0
        out["pos"][b, 0] = cache_len[b]
        out["score"][b, 0] = np.float32(0.0)
        index_of = {(): 0}
        for i, (ranks, score) in enumerate(nodes, start=1):
            d = len(ranks)
            index_of[ranks] = i
            out["node_tok"][b, i] = tok[b, d - 1, ranks[-1]]
            out["parent"][b, i] = index_of[ranks[:-1]]
            out["depth"][b, i] = d
            out["pos"][b, i] = cache_len[b] + d
            out["score"][b, i] = score
        n = 1 + len(nodes)
        out["n_nodes"][b] = n
        for i in range(n):
            j = i
            while j >= 0:
                out["mask"][b, i, j >> 5] |= np.uint32(1 << (j & 31))
                j = out["parent"][b, j]
    return out


def _best_first(logp_b: np.ndarray, budget: int):
    """Pop up to ``budget`` rank paths in key order. Returns [(ranks, score)]."""
    D, K = logp_b.shape
    picked = []
    if budget <= 0:
        return picked
    # heap item: (-score, depth, ranks, score, parent_score)
    zero = np.float32(0.0)
    s0 = np.float32(zero + logp_b[0, 0])
    heap = [(-s0, 1, (0,), s0, zero)]
    while heap and len(picked) < budget:
        _, d, ranks, score, parent_score = heapq.heappop(heap)
        picked.append((ranks, score))
        if d < D:  # first child: append rank 0 at depth d + 1
            cs = np.float32(score + logp_b[d, 0])
            heapq.heappush(heap, (-cs, d + 1, ranks + (0,), cs, score))
        r = ranks[-1]
        if r + 1 < K:  # next sibling under the same parent
            ss = np.float32(parent_score + logp_b[d - 1, r + 1])
            heapq.heappush(heap, (-ss, d, ranks[:-1] + (r + 1,), ss, parent_score))
    return picked


# ---------------------------------------------------------------------------
# a2: MLA-absorb tree-verify attention
# ---------------------------------------------------------------------------


def widen(x: np.ndarray, dtype: str) -> np.ndarray:
    """Stored values (float32, bfloat16 bit patterns in uint16, or float64 for
    exact pins) as float64."""
    if dtype == "f64":
        return np.asarray(x, np.float64)
    if dtype == "f32":
        return np.asarray(x, np.float32).astype(np.float64)
    u = np.ascontiguousarray(x, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def visible_keys(L_b: int, n_b: int, mask_row: np.ndarray) -> np.ndarray:
    """Key indices (relative to the request's first pool row) a tree node sees:
    every committed cache row [0, L_b) and tree row L_b + t for each node t < n_b
    whose bit is set in the node's visibility mask (first page, "Broader
    Context": tree-verify attention "with visibility masking")."""
    tree = [L_b + t for t in range(n_b) if (int(mask_row[t >> 5]) >> (t & 31)) & 1]
    return np.concatenate([np.arange(L_b, dtype=np.int64), np.array(tree, np.int64)])


def verify_attn(q, kv, cache_off, cache_len, mask, n_nodes, H, d_l, d_r, scale, dtype, rows=None):
    """MLA-absorb attention of every tree node's heads over its visible keys.

    Absorbed MLA (first page, "Broader Context"; capstone page "Context and
    Motivation"): each pool row is [c (d_l latent) ; k_pe (d_r rope)], the key
    is the whole row and the value is the latent c, shared by all heads.
    For request b, node i < n_nodes[b], head h:
        s_j = scale * sum_c q[b,i,h,c] * kv[off_b + j, c]     over visible j
        out = sum_j softmax(s)_j * kv[off_b + j, :d_l]
        lse = ln sum_j exp(s_j)
    computed in float64 from the stored inputs. Pad rows: out 0, lse -inf.
    ``rows``: optional list of (b, i) to compute (others left 0 / -inf).
    Returns (out [B, N, H, d_l] float64, lse [B, N, H] float64).
    """
    B, N = q.shape[0], q.shape[1]
    d_qk = d_l + d_r
    out = np.zeros((B, N, H, d_l), np.float64)
    lse = np.full((B, N, H), -np.inf, np.float64)
    want = None if rows is None else {(int(b), int(i)) for b, i in rows}
    for b in range(B):
        n_b = int(n_nodes[b])
        L_b = int(cache_len[b])
        off = int(cache_off[b])
        todo = [i for i in range(n_b) if want is None or (b, i) in want]
        if not todo:
            continue
        keys = widen(kv[off:off + L_b + n_b], dtype)  # [L_b + n_b, d_qk]
        for i in todo:
            vis = visible_keys(L_b, n_b, mask[b, i])
            Kv = keys[vis]  # [n_vis, d_qk]
            Q = widen(q[b, i], dtype).reshape(H, d_qk)
            s = scale * (Q @ Kv.T)  # [H, n_vis]
            m = s.max(axis=1, keepdims=True)
            e = np.exp(s - m)
            z = e.sum(axis=1, keepdims=True)
            out[b, i] = (e / z) @ Kv[:, :d_l]
            lse[b, i] = (m + np.log(z))[:, 0]
    return out, lse


# ---------------------------------------------------------------------------
# a3 + a4: greedy accept walk and latent-KV compaction
# ---------------------------------------------------------------------------


def widen_logits(x: np.ndarray, dtype: str) -> np.ndarray:
    """Logits as float32 (bf16 patterns widened exactly)."""
    if dtype == "f32":
        return np.asarray(x, np.float32)
    u = np.ascontiguousarray(x, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32)


def row_argmax(logits_f32: np.ndarray) -> np.ndarray:
    """Greedy target token of every verify row: index of the largest logit,
    the lowest index among equals (READING: the pages fix no tie rule)."""
    return np.argmax(logits_f32, axis=-1).astype(np.int32)


def accept_walk(am_b, node_tok_b, parent_b, n_b):
    """Greedy tree accept for one request (first page, "Broader Context":
    greedy tree-accept kernel; capstone page: the target's prediction at the
    last accepted node is the bonus token).

    Start at the root; while some child c of the current node carries the token
    the target predicts there (am[cur]), move to it (the lowest such c);
    stop otherwise. Returns the accepted node path, root first."""
    path = [0]
    cur = 0
    while True:
        nxt = -1
        for c in range(1, n_b):
            if parent_b[c] == cur and node_tok_b[c] == am_b[cur]:
                nxt = c
                break
        if nxt < 0:
            return path
        path.append(nxt)
        cur = nxt


def accept_compact(logits, logits_dtype, node_tok, parent, n_nodes, kv, cache_off, cache_len, cache_cap,
                   n_layers=1, layer_stride_rows=0):
    """Accept + compaction for every request.

    a = len(path) - 1 accepted drafted nodes; committed tokens are the a
    accepted node tokens followed by the bonus token am[path[a]].
    Compaction (first page, "Broader Context": KV cache with post-verify
    compaction): the latent rows of the accepted nodes move, in path order, to
    the contiguous cache right after the committed rows:
        kv[off + L + j] <- kv[off + L + path[j]]   for j = 0..a
    (all rows read before any is written), on every layer; cache_len += a + 1.

    ``kv`` is modified in place (numpy array of rows). Returns a dict with
    am [B, N], acc_len [B], acc_nodes [B, N], out_tok [B, N], bonus [B],
    cache_len [B] (new), status [B]. Requests with n_nodes = 0 are skipped
    (acc_len 0, bonus -1, nothing copied); a request whose L + n exceeds its
    capacity gets status ERR_CAPACITY and is skipped the same way.
    """
    B, N = node_tok.shape
    lf = widen_logits(logits, logits_dtype)
    am = np.full((B, N), -1, np.int32)
    res = {
        "acc_len": np.zeros(B, np.int32),
        "acc_nodes": np.full((B, N), -1, np.int32),
        "out_tok": np.full((B, N), -1, np.int32),
        "bonus": np.full(B, -1, np.int32),
        "cache_len": np.asarray(cache_len, np.int32).copy(),
        "status": np.zeros(B, np.int32),
    }
    for b in range(B):
        n_b = int(n_nodes[b])
        if n_b > 0:
            am[b, :n_b] = row_argmax(lf[b, :n_b])
        if n_b <= 0:
            continue
        L_b = int(cache_len[b])
        if L_b + n_b > int(cache_cap[b]):
            res["status"][b] = ERR_CAPACITY
            continue
        path = accept_walk(am[b], node_tok[b], parent[b], n_b)
        a = len(path) - 1
        res["acc_len"][b] = a
        res["acc_nodes"][b, :a + 1] = path
        res["out_tok"][b, :a] = [node_tok[b, p] for p in path[1:]]
        res["out_tok"][b, a] = am[b, path[a]]
        res["bonus"][b] = am[b, path[a]]
        base = int(cache_off[b]) + L_b
        for layer in range(n_layers):
            lb = base + layer * int(layer_stride_rows)
            src = np.array([kv[lb + p].copy() for p in path])  # read everything first
            for j in range(a + 1):
                kv[lb + j] = src[j]
        res["cache_len"][b] = L_b + a + 1
    res["am"] = am
    return res


# ---------------------------------------------------------------------------
# drafter proposals: per-depth log-softmax + top-k over the vocabulary
# ---------------------------------------------------------------------------


def drafter_topk(logits, K):
    """Per-row drafter proposals, the input contract of the tree build.

    Source: capstone page, "The Oracle Drafter" (the drafter hands the tree
    builder, for every depth, log-probabilities and token ids of its best
    candidates, sorted best first); AR page, "The Broader Context" (the
    draft tree is built from the drafter's per-depth top-k).

    logits: [R, V] float (bf16 already widened exactly); K <= V.
    Returns (logp [R, K] float32, tok [R, K] int32, status [R] int32):
      tok[r] = the K indices of the largest logits, largest first;
               READING: equal values are ordered by lower index first.
      logp[r][k] = logits[r][tok[r][k]] - logsumexp(logits[r]), computed in
               float64 and rounded to float32 once.
      status OK, or ERR_INPUT for a row with a non-finite logit (READING:
      that row's outputs are tok -1, logp -inf).
    """
    x = np.asarray(logits, dtype=np.float64)
    R, V = x.shape
    logp = np.full((R, K), -np.inf, np.float32)
    tok = np.full((R, K), -1, np.int32)
    status = np.full(R, OK, np.int32)
    for r in range(R):
        z = x[r]
        if not np.all(np.isfinite(z)):
            status[r] = ERR_INPUT
            continue
        m = z.max()
        lse = m + math.log(np.exp(z - m).sum())
        order = np.lexsort((np.arange(V), -z))[:K]  # value descending, then index ascending
        tok[r] = order.astype(np.int32)
        logp[r] = (z[order] - lse).astype(np.float32)
    return logp, tok, status


# ---------------------------------------------------------------------------
# target LM head folded into the accept argmax
# ---------------------------------------------------------------------------


def lmhead_logits(hidden, w_vocab, v_chunk=None):
    """The target's logits from its final hidden states: z[r][v] = sum over c of
    hidden[r][c] * w_vocab[v][c], in float64 from the stored values (bf16
    already widened exactly). ``v_chunk``: evaluate the product one slice of
    the vocabulary at a time (each logit is still one float64 dot product;
    only the memory of the widened head is bounded).

    Source: AR page, "What the Message Actually Says" (the greedy token of a
    verify row is the argmax of the target's logits, checked exactly);
    "the_validation_pivot", "Assumptions Embedded in This Message" (Kimi K2.6:
    hidden size 7168; the tests' tiny model: hidden 64, vocabulary 400).
    hidden: [R, d]; w_vocab: [V, d] (one row per token). Returns [R, V]."""
    h = np.asarray(hidden, dtype=np.float64)
    V = np.shape(w_vocab)[0]
    step = V if v_chunk is None else int(v_chunk)
    z = np.empty((h.shape[0], V), np.float64)
    for v0 in range(0, V, step):
        z[:, v0:v0 + step] = h @ np.asarray(w_vocab[v0:v0 + step], dtype=np.float64).T
    return z


def lmhead_argmax(hidden, w_vocab):
    """Greedy target token of every verify row without materialised logits:
    the lowest v attaining the float64 maximum of lmhead_logits (the tie rule
    is row_argmax's). Returns am [R] int32."""
    return np.argmax(lmhead_logits(hidden, w_vocab), axis=-1).astype(np.int32)


# READING (the pages fix no precision for the head): a GPU evaluates the dot
# products in float32 with every bf16 x bf16 product exact (16 significant bits
# fit float32's 24) and every addition off by at most u relative, in an order
# of its own. If no product passes through more than n roundings on its way
# into the sum, the classical bound on floating-point summation (Higham,
# "Accuracy and Stability of Numerical Algorithms", section 4.2) gives
# |z32 - z| <= gamma(n) * sum over c of |h_c w_vc|, gamma(n) = n u / (1 - n u).
# n = d - 1 covers every order; an evaluation that adds 16-product steps one
# after another has n <= 15 + d / 16. u = 2^-22: twice float32's truncation
# unit, a margin for tensor-core accumulators that align the products of one
# step to the largest before adding them.
LMHEAD_U = 2.0 ** -22


def lmhead_f32_error_bound(hidden, w_vocab, depth=None, v_chunk=None):
    """Per row, the largest over v of the float32 evaluation bound above, for
    at most ``depth`` roundings per product (default d - 1: any order).
    Returns [R] float64."""
    h = np.abs(np.asarray(hidden, dtype=np.float64))
    n = max(h.shape[1] - 1, 0) if depth is None else int(depth)
    gamma = n * LMHEAD_U / (1.0 - n * LMHEAD_U)
    V = np.shape(w_vocab)[0]
    step = V if v_chunk is None else int(v_chunk)
    top = np.zeros(h.shape[0], np.float64)
    for v0 in range(0, V, step):
        top = np.maximum(top, (h @ np.abs(np.asarray(w_vocab[v0:v0 + step], dtype=np.float64)).T).max(axis=-1))
    return gamma * top


def lmhead_valid_argmax(hidden, w_vocab, depth=None, v_chunk=None):
    """The tokens a float32 evaluation within the bound may pick for each row:
    every v with z[v] >= max(z) - 2 * bound (a pick g has z[g] >= z32[g] - bound
    >= z32[am] - bound >= z[am] - 2 * bound). Returns (am [R] int32, valid: a
    list of R sorted int32 arrays, each holding am)."""
    z = lmhead_logits(hidden, w_vocab, v_chunk)
    bound = lmhead_f32_error_bound(hidden, w_vocab, depth, v_chunk)
    am = np.argmax(z, axis=-1).astype(np.int32)
    top = z.max(axis=-1)
    valid = [np.flatnonzero(z[r] >= top[r] - 2.0 * bound[r]).astype(np.int32) for r in range(z.shape[0])]
    return am, valid
