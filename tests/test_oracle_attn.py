"""Pins for the oracle's MLA-absorb tree-verify attention against independent
statements of the same quantity: materialised multi-head attention with random
up-projections (the absorption identity), causal scaled-dot-product attention
for a chain tree, plain decode attention for a single row, a two-key closed
form, and a pure-Python loop that finds visible keys from parent pointers."""
import math

import numpy as np
import pytest
import torch

from oracle import build_tree, verify_attn
from ddtree_speculative_decode_b200 import synth


def _chain_inputs(rng, L, n, H, d_l, d_r):
    d_qk = d_l + d_r
    kv = rng.standard_normal((L + n, d_qk)).astype(np.float32)
    q = rng.standard_normal((1, n, H, d_qk)).astype(np.float32)
    mask = np.zeros((1, n, (n + 31) // 32), np.uint32)
    for i in range(n):
        for j in range(i + 1):
            mask[0, i, j >> 5] |= np.uint32(1 << (j & 31))
    return kv, q, mask


def test_absorption_identity():
    """Absorbed MLA equals materialised MHA: with k_nope = W_UK c, v = W_UV c
    and q_lat = W_UK^T q_nope, the materialised head output is W_UV applied to
    the latent-space output."""
    rng = np.random.default_rng(0)
    H, d_nope, d_l, d_r, d_v, L, n = 3, 8, 24, 6, 10, 9, 4
    W_UK = rng.standard_normal((H, d_nope, d_l))
    W_UV = rng.standard_normal((H, d_v, d_l))
    c = rng.standard_normal((L + n, d_l))
    k_pe = rng.standard_normal((L + n, d_r))
    q_nope = rng.standard_normal((n, H, d_nope))
    q_pe = rng.standard_normal((n, H, d_r))
    scale = 1.0 / math.sqrt(d_nope + d_r)
    # tree: a chain plus a side branch (node 3 is a child of node 1)
    parents = [-1, 0, 1, 1]
    vis = []
    for i in range(n):
        s, j = set(), i
        while j >= 0:
            s.add(j)
            j = parents[j]
        vis.append(s)
    mask = np.zeros((1, n, 1), np.uint32)
    for i in range(n):
        for j in vis[i]:
            mask[0, i, 0] |= np.uint32(1 << j)
    # materialised MHA
    ref = np.zeros((n, H, d_v))
    for i in range(n):
        keys = list(range(L)) + [L + t for t in sorted(vis[i])]
        for h in range(H):
            kn = c[keys] @ W_UK[h].T  # [nk, d_nope]
            s = scale * (kn @ q_nope[i, h] + k_pe[keys] @ q_pe[i, h])
            p = np.exp(s - s.max())
            p /= p.sum()
            ref[i, h] = p @ (c[keys] @ W_UV[h].T)
    q_lat = np.einsum("nhd,hdl->nhl", q_nope, W_UK)
    q = np.concatenate([q_lat, q_pe], axis=-1)[None]
    kv = np.concatenate([c, k_pe], axis=-1)
    out, _ = _verify64(q, kv, L, n, mask, H, d_l, d_r, scale)
    got = np.einsum("hvl,nhl->nhv", W_UV, out[0])
    np.testing.assert_allclose(got, ref, rtol=1e-10, atol=1e-10)


def _verify64(q, kv, L, n, mask, H, d_l, d_r, scale):
    """The oracle on float64 data, so the pin is not limited by rounding."""
    return verify_attn(q, kv, np.array([0]), np.array([L]), mask, np.array([n]), H, d_l, d_r, scale, "f64")


@pytest.mark.parametrize("L,n", [(0, 5), (7, 1), (13, 6), (3, 40)])
def test_chain_tree_equals_causal_sdpa(L, n):
    rng = np.random.default_rng(L * 31 + n)
    H, d_l, d_r = 2, 16, 4
    kv, q, mask = _chain_inputs(rng, L, n, H, d_l, d_r)
    scale = 0.37
    out, lse = verify_attn(q, kv, np.array([0]), np.array([L]), mask, np.array([n]), H, d_l, d_r, scale, "f32")
    # torch SDPA in float64 with an explicit causal-over-(cache || chain) mask
    K = torch.from_numpy(kv.astype(np.float64))  # [L+n, d_qk]
    Q = torch.from_numpy(q[0].astype(np.float64)).permute(1, 0, 2)  # [H, n, d_qk]
    allowed = torch.zeros(n, L + n, dtype=torch.bool)
    for i in range(n):
        allowed[i, :L + i + 1] = True
    ref = torch.nn.functional.scaled_dot_product_attention(
        Q, K.expand(H, -1, -1), K[:, :d_l].expand(H, -1, -1), attn_mask=allowed, scale=scale)
    np.testing.assert_allclose(out[0], ref.permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-12)
    S = (Q @ K.T) * scale
    S = S.masked_fill(~allowed, float("-inf"))
    np.testing.assert_allclose(lse[0], torch.logsumexp(S, -1).T.numpy(), rtol=1e-12, atol=1e-12)


def test_single_row_is_decode_attention():
    rng = np.random.default_rng(2)
    H, d_l, d_r, L = 4, 32, 8, 50
    kv, q, mask = _chain_inputs(rng, L, 1, H, d_l, d_r)
    out, _ = verify_attn(q, kv, np.array([0]), np.array([L]), mask, np.array([1]), H, d_l, d_r, 0.2, "f32")
    K = torch.from_numpy(kv.astype(np.float64))
    Q = torch.from_numpy(q[0, 0].astype(np.float64))  # [H, d_qk]
    ref = torch.softmax(0.2 * Q @ K.T, -1) @ K[:, :d_l]
    np.testing.assert_allclose(out[0, 0], ref.numpy(), rtol=1e-12, atol=1e-12)


def test_two_key_closed_form():
    # d_qk = 1, one cached key plus the root: p = sigmoid(s1 - s2)
    kv = np.array([[1.5], [-0.5]], np.float32)
    q = np.array([[[[2.0]]]], np.float32)
    out, lse = verify_attn(q, kv, np.array([0]), np.array([1]), np.ones((1, 1, 1), np.uint32),
                           np.array([1]), 1, 1, 0, 0.5, "f32")
    s1, s2 = 0.5 * 2.0 * 1.5, 0.5 * 2.0 * -0.5
    p1 = 1.0 / (1.0 + math.exp(s2 - s1))
    assert abs(out[0, 0, 0, 0] - (p1 * 1.5 + (1 - p1) * -0.5)) < 1e-15
    assert abs(lse[0, 0, 0] - math.log(math.exp(s1) + math.exp(s2))) < 1e-15


def test_tree_matches_python_loops_with_parent_walk():
    """Non-chain tree from the builder; visible keys found by walking parent
    pointers in pure Python, scores and softmax by scalar loops."""
    s = synth.custom(B=2, D=3, K=3, N=11, H=2, d_l=8, d_r=4, V=50, L=(5, 2), dtype="f32", seed=3)
    x = synth.make_step(s)
    t = build_tree(x.logp, x.tok, x.root_tok, x.cache_len, s.N)
    out, lse = verify_attn(x.q, x.kv, x.cache_off, x.cache_len, t["mask"], t["n_nodes"], s.H, s.d_l, s.d_r,
                           s.scale, "f32")
    for b in range(s.B):
        off, L, n = int(x.cache_off[b]), int(x.cache_len[b]), int(t["n_nodes"][b])
        for i in range(n):
            anc, j = [], i
            while j >= 0:
                anc.append(j)
                j = int(t["parent"][b, j])
            keys = list(range(L)) + [L + a for a in sorted(anc)]
            for h in range(s.H):
                sc = []
                for k in keys:
                    acc = 0.0
                    for c in range(s.d_qk):
                        acc += float(x.q[b, i, h, c]) * float(x.kv[off + k, c])
                    sc.append(s.scale * acc)
                m = max(sc)
                e = [math.exp(v - m) for v in sc]
                z = sum(e)
                for c in range(s.d_l):
                    ref = sum(e[u] * float(x.kv[off + keys[u], c]) for u in range(len(keys))) / z
                    assert abs(out[b, i, h, c] - ref) < 1e-12
                assert abs(lse[b, i, h] - (m + math.log(z))) < 1e-12
        # pad rows
        assert np.all(out[b, n:] == 0) and np.all(np.isneginf(lse[b, n:]))


def test_bf16_widening_is_exact():
    x = np.array([1.5, -2.25, 0.0078125, 3.0e38, -1.0e-38], np.float32)
    bits = synth.f32_to_bf16_bits(x[:3])
    from oracle import widen
    np.testing.assert_array_equal(widen(bits, "bf16"), x[:3].astype(np.float64))
    # round to nearest even at a tie: 1 + 2^-8 is halfway between 1 and 1 + 2^-7
    t = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8], np.float32)
    np.testing.assert_array_equal(widen(synth.f32_to_bf16_bits(t), "bf16"), [1.0, 1.0 + 2.0 ** -6])
