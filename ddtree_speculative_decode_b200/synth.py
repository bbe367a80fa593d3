"""Seeded synthetic inputs for one DDTree tree-verify step.

This module only draws random numbers and lays them out in the buffers the
tree-verify path consumes. It holds none of the method's arithmetic (no tree
build, no attention, no argmax walk): the same arrays feed the CPU oracle and
the CUDA library, so both sides always see identical bytes.

Workloads restate the shapes of the pages' subject (Kimi K2.6 MLA: 64 heads,
512-d compressed latent + 64-d RoPE key, vocab 163840; "ddtree_speculative_
decode_test_capstone", section "What the Test Validated": a drafter hands the
tree builder per-depth log-probs and token ids, block size = budget + 1).
The pages use a private tiny-model bundle and no public dataset, so every
input here is synthetic:

* drafter: per depth, logits ~ N(0, sigma) over the vocab, log_softmax in
  float64 rounded to float32, top-k by value (ties to the lower id), sorted
  descending. This stands in for a drafter and produces the tree build's
  inputs; it is the workload's recipe, not a side of any parity check (the
  drafter-proposal kernel is checked on raw logits against the oracle's own
  drafter_topk, which shares nothing with this function);
* latent KV rows and queries ~ N(0, 1), KV optionally scaled (0.1 on the
  Kimi-shaped workloads), rounded to the storage dtype (bf16 round-to-nearest-
  even, or float32);
* target logits ~ N(0, 1); for each tree node in index order a uniform draw u,
  and if u < p and the node has children, +bias on the token of one child
  chosen uniformly (so accepted paths are non-contiguous in node index);
* the target's LM-head inputs and a tiny decoder's random weights, for the
  steps around the path (lmhead_inputs, tiny_mla_weights).

``N(0, s)`` is read as standard deviation ``s``.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

# ---------------------------------------------------------------------------
# storage helpers (format conversion only)
# ---------------------------------------------------------------------------


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round-to-nearest-even); returns the
    16-bit patterns as uint16. Inputs here are finite."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rnd = ((b >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((b + rnd) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(u: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float32."""
    return (np.ascontiguousarray(u, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# ---------------------------------------------------------------------------
# workload description
# ---------------------------------------------------------------------------


@dataclasses.dataclass(frozen=True)
class Shape:
    """One tree-verify workload.

    B requests; drafter depth D, top-k K; N = tree budget counted in verify
    rows including the root (N - 1 drafted nodes); H heads; latent dim d_l,
    RoPE dim d_r (QK uses d_l + d_r, V uses the first d_l); vocab V.
    """

    name: str
    B: int
    D: int
    K: int
    N: int
    H: int
    d_l: int
    d_r: int
    V: int
    scale: float
    dtype: str  # "f32" or "bf16" (storage of q, kv, logits)
    L: tuple  # per-request committed cache length
    drafter_sigma: float
    kv_scale: float
    accept_p: float
    accept_bias: float
    seed: int

    @property
    def d_qk(self) -> int:
        return self.d_l + self.d_r

    @property
    def W(self) -> int:
        return (self.N + 31) // 32


def _cache_lengths(seed: int, B: int, lo: int, hi: int) -> tuple:
    rng = np.random.default_rng(np.random.SeedSequence([seed, 7]))
    return tuple(int(v) for v in rng.integers(lo, hi + 1, size=B))


def tiny_f32() -> Shape:
    """Tiny fp32 step, batch 1: 4 heads, latent 64 + rope 16, cache 32 rows,
    drafter depth 4 x top-2 over vocab 256, budget 8 rows, scale 1/sqrt(24)."""
    return Shape("tiny-f32", B=1, D=4, K=2, N=8, H=4, d_l=64, d_r=16, V=256,
                 scale=1.0 / math.sqrt(24.0), dtype="f32", L=(32,), drafter_sigma=2.0,
                 kv_scale=1.0, accept_p=0.7, accept_bias=5.0, seed=1001)


def kimi_1req() -> Shape:
    """Kimi-K2.6-shaped single request: 64 heads, 512 + 64 latent, bf16,
    cache 4096 rows, depth 8 x top-8 over vocab 163840, budget 64 rows."""
    return Shape("kimi-1req-L4096-N64", B=1, D=8, K=8, N=64, H=64, d_l=512, d_r=64, V=163840,
                 scale=1.0 / math.sqrt(192.0), dtype="bf16", L=(4096,), drafter_sigma=3.0,
                 kv_scale=0.1, accept_p=0.8, accept_bias=6.0, seed=1002)


def kimi_16req_ragged() -> Shape:
    """Batched serving step: 16 requests, cache lengths uniform in
    [1024, 8192], depth 6 x top-6, budget 32 rows per request."""
    return Shape("kimi-16req-ragged-N32", B=16, D=6, K=6, N=32, H=64, d_l=512, d_r=64, V=163840,
                 scale=1.0 / math.sqrt(192.0), dtype="bf16", L=_cache_lengths(1003, 16, 1024, 8192),
                 drafter_sigma=2.0, kv_scale=0.1, accept_p=0.7, accept_bias=5.0, seed=1003)


def kimi_4req_32k() -> Shape:
    """Long-context step: 4 requests with 32768 cached rows each, depth 16 x
    top-8, budget 128 rows per request, +6 bias at 85 % of nodes."""
    return Shape("kimi-4req-L32768-N128", B=4, D=16, K=8, N=128, H=64, d_l=512, d_r=64, V=163840,
                 scale=1.0 / math.sqrt(192.0), dtype="bf16", L=(32768,) * 4, drafter_sigma=2.0,
                 kv_scale=0.1, accept_p=0.85, accept_bias=6.0, seed=1004)


def kimi_sweep(B: int, N: int, L: int) -> Shape:
    """One point of the Kimi-shaped sweep: depth 8, top-k = min(16, N / 4)."""
    return Shape(f"kimi-sweep-B{B}-N{N}-L{L}", B=B, D=8, K=min(16, max(1, N // 4)), N=N, H=64,
                 d_l=512, d_r=64, V=163840, scale=1.0 / math.sqrt(192.0), dtype="bf16", L=(L,) * B,
                 drafter_sigma=2.0, kv_scale=0.1, accept_p=0.7, accept_bias=5.0,
                 seed=2000 + 100 * B + N + L % 97)


def custom(name: str = "custom", *, B=1, D=3, K=2, N=8, H=2, d_l=64, d_r=16, V=64, dtype="f32",
           L=(16,), scale: Optional[float] = None, drafter_sigma=2.0, kv_scale=1.0, accept_p=0.7,
           accept_bias=5.0, seed=7) -> Shape:
    """Small hand-sized workload for edge-case tests."""
    if scale is None:
        scale = 1.0 / math.sqrt(float(d_l + d_r))
    L = tuple(int(x) for x in L)
    assert len(L) == B
    return Shape(name, B=B, D=D, K=K, N=N, H=H, d_l=d_l, d_r=d_r, V=V, scale=scale, dtype=dtype,
                 L=L, drafter_sigma=drafter_sigma, kv_scale=kv_scale, accept_p=accept_p,
                 accept_bias=accept_bias, seed=seed)


NAMED = {
    "tiny-f32": tiny_f32,
    "kimi-1req": kimi_1req,
    "kimi-16req": kimi_16req_ragged,
    "kimi-4req-32k": kimi_4req_32k,
}

# ---------------------------------------------------------------------------
# draws
# ---------------------------------------------------------------------------


def _rng(seed: int, *path: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([seed, *path]))


def _store(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "f32":
        return np.ascontiguousarray(x, dtype=np.float32)
    return f32_to_bf16_bits(x.astype(np.float32))


@dataclasses.dataclass
class StepInputs:
    """Host arrays for one step. ``kv`` / ``q`` / logits are float32 arrays for
    dtype f32 and uint16 bf16 bit patterns for dtype bf16."""

    shape: Shape
    root_tok: np.ndarray  # [B] i32
    cache_len: np.ndarray  # [B] i32
    cache_off: np.ndarray  # [B] i64, first pool row of request b
    cache_cap: np.ndarray  # [B] i32, rows owned by request b
    logp: np.ndarray  # [B, D, K] f32, sorted descending per depth
    tok: np.ndarray  # [B, D, K] i32
    kv: np.ndarray  # [rows, d_qk]
    q: np.ndarray  # [B, N, H, d_qk]


def drafter_topk(rng: np.random.Generator, D: int, K: int, V: int, sigma: float):
    """Per-depth drafter proposals: log_softmax of N(0, sigma) logits (float64,
    rounded to float32), top-K by value with ties to the lower id."""
    logp = np.empty((D, K), np.float32)
    tok = np.empty((D, K), np.int32)
    for d in range(D):
        z = rng.standard_normal(V) * sigma
        m = z.max()
        ls = (z - m) - math.log(np.exp(z - m).sum())
        ls32 = ls.astype(np.float32)
        # stable order: value descending, id ascending
        idx = np.lexsort((np.arange(V), -ls32.astype(np.float64)))[:K]
        logp[d] = ls32[idx]
        tok[d] = idx.astype(np.int32)
    return logp, tok


def make_step(shape: Shape, requests: Optional[list] = None, rows: bool = True) -> StepInputs:
    """Draw all pre-tree inputs of one step.

    ``requests`` (optional) restricts the draws to a subset of request ids; the
    per-request streams are independent, so a subset sees the same values as a
    full draw. ``rows=False`` skips the latent rows and queries (kv and q are
    then empty arrays of the right shape's dtype): the other draws are the same.
    """
    s = shape
    reqs = list(range(s.B)) if requests is None else list(requests)
    B = len(reqs)
    L = np.array([s.L[b] for b in reqs], np.int32)
    cap = L + s.N
    off = np.zeros(B, np.int64)
    off[1:] = np.cumsum(cap[:-1].astype(np.int64))
    n_rows = int(cap.astype(np.int64).sum())
    d_qk = s.d_qk
    kv = np.zeros((n_rows if rows else 0, d_qk), np.float32 if s.dtype == "f32" else np.uint16)
    q = np.zeros((B if rows else 0, s.N, s.H, d_qk), kv.dtype)
    logp = np.zeros((B, s.D, s.K), np.float32)
    tok = np.zeros((B, s.D, s.K), np.int32)
    root = np.zeros(B, np.int32)
    for j, b in enumerate(reqs):
        r = _rng(s.seed, 1, b)
        root[j] = int(r.integers(0, s.V))
        logp[j], tok[j] = drafter_topk(_rng(s.seed, 2, b), s.D, s.K, s.V, s.drafter_sigma)
        if not rows:
            continue
        rk = _rng(s.seed, 3, b)
        blk = rk.standard_normal((int(L[j]) + s.N, d_qk), dtype=np.float32) * np.float32(s.kv_scale)
        kv[off[j]:off[j] + L[j] + s.N] = _store(blk, s.dtype)
        rq = _rng(s.seed, 4, b)
        q[j] = _store(rq.standard_normal((s.N, s.H, d_qk), dtype=np.float32), s.dtype)
    return StepInputs(shape=s, root_tok=root, cache_len=L.copy(), cache_off=off, cache_cap=cap.astype(np.int32),
                      logp=logp, tok=tok, kv=kv, q=q)


def target_logits(shape: Shape, parent: np.ndarray, node_tok: np.ndarray, n_nodes: np.ndarray,
                  requests: Optional[list] = None) -> np.ndarray:
    """Target-model logits for every verify row, [B, N, V].

    ``parent`` / ``node_tok`` / ``n_nodes`` describe the tree the rows belong to
    (they only decide which token gets the acceptance bias).
    """
    s = shape
    reqs = list(range(s.B)) if requests is None else list(requests)
    out = np.empty((len(reqs), s.N, s.V), np.float32 if s.dtype == "f32" else np.uint16)
    for j, b in enumerate(reqs):
        r = _rng(s.seed, 5, b)
        z = r.standard_normal((s.N, s.V), dtype=np.float32)
        rb = _rng(s.seed, 6, b)
        n = int(n_nodes[j])
        for i in range(s.N):
            u = rb.random()
            pick = rb.random()
            if i >= n:
                continue
            kids = [c for c in range(n) if parent[j, c] == i]
            if kids and u < s.accept_p:
                c = kids[min(len(kids) - 1, int(pick * len(kids)))]
                z[i, int(node_tok[j, c])] += np.float32(s.accept_bias)
        out[j] = _store(z, s.dtype)
    return out


def lmhead_inputs(shape: Shape, parent: np.ndarray, node_tok: np.ndarray, n_nodes: np.ndarray, d_model: int,
                  requests: Optional[list] = None, w_vocab: Optional[np.ndarray] = None):
    """Inputs of the target's LM head for every verify row: the head's weights
    w_vocab [V, d_model] (one row per token, N(0, 1 / d_model), so logits have
    unit scale like target_logits') and final hidden states hidden
    [B, N, d_model] (N(0, 1)). At the same fraction of nodes as target_logits,
    a uniformly chosen child's token t gets the acceptance bias: hidden row i
    moves by bias * w_t / |w_t|^2 (w_t as stored), which raises its logit for t
    by the bias before rounding. Returns (hidden, w_vocab, planted [B, N] i32:
    the planted token, or -1), hidden and w_vocab in the shape's dtype.
    ``w_vocab`` (optional, [V, d_model] as stored): use this head instead of
    drawing one (several workloads against one large head)."""
    s = shape
    reqs = list(range(s.B)) if requests is None else list(requests)
    # drawn in row blocks (the same stream as one draw) so a Kimi-sized head
    # (163840 x 7168) never needs more than a block of float32 temporaries
    if w_vocab is not None:
        w = w_vocab
        assert w.shape == (s.V, d_model)
    else:
        rw = _rng(s.seed, 7)
        w = np.empty((s.V, d_model), np.float32 if s.dtype == "f32" else np.uint16)
        scale = np.float32(math.sqrt(d_model))
        for v0 in range(0, s.V, 8192):
            blk = rw.standard_normal((min(8192, s.V - v0), d_model), dtype=np.float32) / scale
            w[v0:v0 + len(blk)] = _store(blk.astype(np.float32), s.dtype)

    def wv(t):  # row t of the head as stored, in float64
        row = w[t:t + 1]
        return (row.astype(np.float64) if s.dtype == "f32" else bf16_bits_to_f32(row).astype(np.float64))[0]

    hidden = np.empty((len(reqs), s.N, d_model), w.dtype)
    planted = np.full((len(reqs), s.N), -1, np.int32)
    for j, b in enumerate(reqs):
        h = _rng(s.seed, 8, b).standard_normal((s.N, d_model)).astype(np.float64)
        rb = _rng(s.seed, 9, b)
        n = int(n_nodes[j])
        for i in range(s.N):
            u = rb.random()
            pick = rb.random()
            if i >= n:
                continue
            kids = [c for c in range(n) if parent[j, c] == i]
            if kids and u < s.accept_p:
                c = kids[min(len(kids) - 1, int(pick * len(kids)))]
                t = int(node_tok[j, c])
                wt = wv(t)
                h[i] += s.accept_bias * wt / float(wt @ wt)
                planted[j, i] = t
        hidden[j] = _store(h.astype(np.float32), s.dtype)
    return hidden, w, planted


def tiny_mla_weights(seed: int = 1234, V: int = 400, d_model: int = 64, n_layers: int = 6, H: int = 4,
                     d_nope: int = 8, d_rope: int = 16, d_latent: int = 64, d_v: int = 16, d_ff: int = 256) -> dict:
    """Random weights of a tiny MLA decoder with the pages' tiny-model sizes
    (hidden 64, 6 layers, vocabulary 400; "the_validation_pivot", section
    "Assumptions Embedded in This Message") and the tiny attention shape (4
    heads, latent 64 + rope 16, scale 1/sqrt(8 + 16)). Every matrix is
    N(0, 1 / fan_in) in float32; the embedding is N(0, 1)."""
    r = _rng(seed, 10)

    def m(*shape):
        return (r.standard_normal(shape) / math.sqrt(shape[-1])).astype(np.float32)

    layers = []
    for _ in range(n_layers):
        layers.append({
            "w_dkv": m(d_latent, d_model),       # latent c = w_dkv x
            "w_kr": m(d_rope, d_model),          # shared rope key, before rotation
            "w_q": m(H, d_nope, d_model),        # per-head no-rope query
            "w_qr": m(H, d_rope, d_model),       # per-head rope query, before rotation
            "w_uk": m(H, d_nope, d_latent),      # key up-projection (absorbed into the query)
            "w_uv": m(H, d_v, d_latent),         # value up-projection (applied to the latent output)
            "w_o": m(d_model, H * d_v),
            "w_1": m(d_ff, d_model),
            "w_2": m(d_model, d_ff),
        })
    return {"embed": r.standard_normal((V, d_model)).astype(np.float32), "layers": layers,
            "w_vocab": m(V, d_model), "V": V, "d_model": d_model, "H": H, "d_nope": d_nope,
            "d_rope": d_rope, "d_latent": d_latent, "d_v": d_v,
            "scale": 1.0 / math.sqrt(d_nope + d_rope)}


def oracle_drafter(golden: np.ndarray, D: int, K: int, sentinel_from: Optional[int] = None):
    """Drafter fixture that proposes a known continuation ("ddtree_speculative_
    decode_test_capstone", section "The Oracle Drafter" and "What the Test
    Validated"): at each depth the golden token sits at rank 0 with log-prob 0,
    then K - 1 distractor ids with strictly decreasing negative log-probs.
    Depths at or past ``sentinel_from`` carry a sentinel id (-7 - depth) at rank
    0 so the target rejects them."""
    logp = np.zeros((D, K), np.float32)
    tok = np.zeros((D, K), np.int32)
    for d in range(D):
        g = int(golden[d]) if d < len(golden) else -1
        if sentinel_from is not None and d >= sentinel_from:
            g = -7 - d
        tok[d, 0] = g
        logp[d, 0] = 0.0
        for k in range(1, K):
            tok[d, k] = 100000 + 97 * d + k  # never a target argmax
            logp[d, k] = np.float32(-1.0 - 0.5 * k)
    return logp, tok
