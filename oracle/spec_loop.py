"""The speculative decoding loop around the tree-verify step, on a tiny MLA
decoder with random weights (test infrastructure, like the rest of oracle/).

Sources: capstone page, "The Oracle Drafter", "What the Test Validated" and
"The Results: A Perfect Validation" (a DDTree loop driven by a drafter that
proposes the golden continuation must reproduce the autoregressive greedy
output token for token, committing a whole block per verify step);
"the_validation_pivot", "The Execution: Remote Validation on PRO 6000" (one
target forward per token for AR against one per block for DDTree) and
"Assumptions Embedded in This Message" (the tiny model: hidden 64, 6 layers,
vocabulary 400); AR page, "The Broader Context" (KV cache with post-verify
compaction).

The model is a plain pre-norm decoder whose attention is absorbed MLA: each
layer caches one latent row [c ; k_pe] per token, and every attention call
-- one new token in the AR loop, a whole draft tree in the DDTree loop --
goes through ddt_oracle.verify_attn on that layer's latent pool, with the
tree's visibility mask. The DDTree loop then uses build_tree and
accept_compact exactly as a user of the library would (all layers compacted
along the accepted path). READINGS: RMS normalisation without weights,
interleaved rotary embedding with base 10000, a ReLU MLP, no biases; logits
are rounded to float32 before the argmax in both loops.
"""
from __future__ import annotations

import numpy as np

from .ddt_oracle import accept_compact, build_tree, row_argmax, verify_attn, widen_logits


def rms(x):
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + 1e-6)


def rope(x, pos, base=10000.0):
    """Rotate consecutive pairs (x[2k], x[2k+1]) of the last axis by
    pos * base^(-2k / d). x: [n, ..., d]; pos: [n]."""
    d = x.shape[-1]
    inv = base ** (-np.arange(0, d, 2, dtype=np.float64) / d)
    ang = np.asarray(pos, np.float64).reshape((-1,) + (1,) * (x.ndim - 1)) * inv
    c, s = np.cos(ang), np.sin(ang)
    xe, xo = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = xe * c - xo * s
    out[..., 1::2] = xe * s + xo * c
    return out


class LatentCache:
    """Per-layer latent pools of one request, stacked at a layer stride so
    accept_compact can compact every layer in one call."""

    def __init__(self, w, capacity):
        self.n_layers = len(w["layers"])
        self.stride = capacity
        self.d_qk = w["d_latent"] + w["d_rope"]
        self.kv = np.zeros((self.n_layers * capacity, self.d_qk), np.float64)
        self.length = 0

    def layer(self, l):
        return self.kv[l * self.stride:(l + 1) * self.stride]


def forward_rows(w, cache: LatentCache, toks, pos, mask):
    """Target forward of n new rows appended after the cache's committed rows:
    row t (token toks[t] at position pos[t]) writes its latent row at cache
    row length + t on every layer and attends to the committed rows plus the
    new rows its mask word(s) select. Returns float64 logits [n, V]."""
    n = len(toks)
    H, dn, dr, dl, dv = w["H"], w["d_nope"], w["d_rope"], w["d_latent"], w["d_v"]
    L = cache.length
    x = w["embed"][np.asarray(toks)].astype(np.float64)
    for li, lw in enumerate(w["layers"]):
        h = rms(x)
        pool = cache.layer(li)
        pool[L:L + n, :dl] = h @ lw["w_dkv"].T.astype(np.float64)
        pool[L:L + n, dl:] = rope(h @ lw["w_kr"].T.astype(np.float64), pos)
        qn = np.einsum("hkd,nd->nhk", lw["w_q"].astype(np.float64), h)
        qr = rope(np.einsum("hkd,nd->nhk", lw["w_qr"].astype(np.float64), h), pos)
        q_lat = np.einsum("hkl,nhk->nhl", lw["w_uk"].astype(np.float64), qn)
        q = np.concatenate([q_lat, qr], axis=-1)[None]  # [1, n, H, dl + dr]
        out, _ = verify_attn(q, pool, np.array([0]), np.array([L]), mask[None], np.array([n]), H, dl, dr,
                             w["scale"], "f64")
        o = np.einsum("hvl,nhl->nhv", lw["w_uv"].astype(np.float64), out[0]).reshape(n, H * dv)
        x = x + o @ lw["w_o"].T.astype(np.float64)
        x = x + np.maximum(rms(x) @ lw["w_1"].T.astype(np.float64), 0.0) @ lw["w_2"].T.astype(np.float64)
    return rms(x) @ w["w_vocab"].T.astype(np.float64)


def _greedy(logits_row):
    return int(row_argmax(widen_logits(logits_row[None], "f32"))[0])


def _one_row(w, cache, tok):
    """The AR step: one token at the next position, seeing the cache and itself."""
    lg = forward_rows(w, cache, [tok], [cache.length], np.ones((1, 1), np.uint32))
    cache.length += 1
    return _greedy(lg[0])


def ar_generate(w, prompt, T, capacity=256):
    """Greedy autoregressive decoding: the prompt row by row (the last prompt
    row's logits give the first token), then one forward per new token.
    Returns (T tokens, the cache)."""
    cache = LatentCache(w, capacity)
    nxt = None
    for t in prompt:
        nxt = _one_row(w, cache, t)
    out = [nxt]
    while len(out) < T:
        out.append(_one_row(w, cache, out[-1]))
    return out, cache


def ddtree_generate(w, prompt, T, drafter, block, K, capacity=256):
    """DDTree greedy decoding: the same prefill, then per verify step a draft
    tree of `block` rows (root = last committed token, block - 1 drafted
    nodes) from the drafter's per-depth top-K, one target forward over the
    tree rows, the greedy accept walk and compaction of every layer.
    drafter(committed, D, K) -> (logp [D, K], tok [D, K]).
    Returns (committed tokens, verify steps, the cache)."""
    cache = LatentCache(w, capacity)
    nxt = None
    for t in prompt:
        nxt = _one_row(w, cache, t)
    committed = [nxt]
    steps = 0
    D = block - 1
    while len(committed) < T:
        lp, tk = drafter(committed, D, K)
        L = cache.length
        tree = build_tree(lp[None], tk[None], np.array([committed[-1]]), np.array([L]), block)
        n = int(tree["n_nodes"][0])
        logits = np.zeros((1, block, w["V"]), np.float64)
        logits[0, :n] = forward_rows(w, cache, tree["node_tok"][0, :n], tree["pos"][0, :n], tree["mask"][0, :n])
        r = accept_compact(logits, "f32", tree["node_tok"], tree["parent"], tree["n_nodes"], cache.kv,
                           np.array([0]), np.array([L], np.int32), np.array([cache.stride], np.int32),
                           n_layers=cache.n_layers, layer_stride_rows=cache.stride)
        a = int(r["acc_len"][0])
        committed += [int(x) for x in r["out_tok"][0, :a + 1]]
        cache.length = int(r["cache_len"][0])
        steps += 1
    return committed, steps, cache
