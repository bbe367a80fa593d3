"""Pins of the oracle's LM-head argmax (the target's head folded into the
accept argmax): closed forms (identity head, one-hot hidden rows), brute force
in exact integer arithmetic, invariances, the tie rule, and the float32 error
bound against float32 evaluations in several summation orders."""
import numpy as np
import pytest

import oracle
from ddtree_speculative_decode_b200 import synth


def _first_max(values):
    best = 0
    for i, v in enumerate(values):
        if v > values[best]:
            best = i
    return best


def _bf16(x):
    return synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(np.asarray(x, np.float32)))


def test_identity_head_is_the_row_argmax():
    rng = np.random.default_rng(1)
    h = rng.integers(-3, 4, size=(40, 9)).astype(np.float32)  # many ties
    am = oracle.lmhead_argmax(h, np.eye(9, dtype=np.float32))
    assert [int(a) for a in am] == [_first_max(list(row)) for row in h]


def test_one_hot_hidden_picks_a_column_of_the_head():
    rng = np.random.default_rng(2)
    w = rng.integers(-5, 6, size=(50, 7)).astype(np.float32)
    w[31] = w[12]  # a duplicated row: column maxima may tie
    am = oracle.lmhead_argmax(np.eye(7, dtype=np.float32), w)
    assert [int(a) for a in am] == [_first_max(list(w[:, c])) for c in range(7)]


def test_integer_inputs_brute_force():
    rng = np.random.default_rng(3)
    for _ in range(20):
        R, d, V = 6, 5, 40
        h = rng.integers(-8, 9, size=(R, d))
        w = rng.integers(-8, 9, size=(V, d))
        am = oracle.lmhead_argmax(h.astype(np.float32), w.astype(np.float32))
        for r in range(R):
            z = [sum(int(h[r, c]) * int(w[v, c]) for c in range(d)) for v in range(V)]
            assert int(am[r]) == _first_max(z)


def test_scaling_and_negation():
    rng = np.random.default_rng(4)
    h = _bf16(rng.standard_normal((16, 32)))
    w = _bf16(rng.standard_normal((300, 32)))
    am = oracle.lmhead_argmax(h, w)
    assert np.array_equal(oracle.lmhead_argmax(2.0 * h, w), am)  # exact in floating point
    assert np.array_equal(oracle.lmhead_argmax(-h, w), np.argmin(h.astype(np.float64) @ w.T.astype(np.float64),
                                                                 axis=-1))


def test_duplicate_rows_tie_to_the_lower_token():
    rng = np.random.default_rng(5)
    w = _bf16(rng.standard_normal((64, 16)))
    h = _bf16(rng.standard_normal((1, 16)))
    w[3] = 10.0 * np.sign(h[0])  # the maximum, twice
    w[11] = w[3]
    assert int(oracle.lmhead_argmax(h, w)[0]) == 3
    am, valid = oracle.lmhead_valid_argmax(h, w)
    assert int(am[0]) == 3 and list(valid[0]) == [3, 11]


def _f32_orders(h, w):
    """float32 evaluations of h @ w.T in four summation orders; each bf16 x bf16
    product is exact in float32."""
    p = h[:, None, :].astype(np.float32) * w[None, :, :].astype(np.float32)
    fwd = np.cumsum(p, axis=-1, dtype=np.float32)[..., -1]
    rev = np.cumsum(p[..., ::-1], axis=-1, dtype=np.float32)[..., -1]
    d = p.shape[-1]
    blocks = np.cumsum(p.reshape(p.shape[0], p.shape[1], d // 16, 16), axis=-1, dtype=np.float32)[..., -1]
    blk = np.cumsum(blocks, axis=-1, dtype=np.float32)[..., -1]
    gemm = (h.astype(np.float32) @ w.T.astype(np.float32)).astype(np.float32)
    return {"forward": fwd, "reverse": rev, "blocked16": blk, "blas": gemm}


def _blocked_depth(d):
    return 15 + d // 16  # 15 roundings inside a 16-product block, then one per later block


@pytest.mark.parametrize("d", [64, 7168])
def test_bound_covers_float32_orders(d):
    rng = np.random.default_rng(6 + d)
    R, V = 4, 256
    h = _bf16(rng.standard_normal((R, d)))
    w = _bf16(rng.standard_normal((V, d)) / np.sqrt(d))
    z = oracle.lmhead_logits(h, w)
    bound = oracle.lmhead_f32_error_bound(h, w)
    am, valid = oracle.lmhead_valid_argmax(h, w)
    orders = _f32_orders(h, w)
    for name, z32 in orders.items():
        err = np.abs(z32.astype(np.float64) - z).max(axis=-1)
        assert np.all(err <= bound), (name, err, bound)
        pick = np.argmax(z32, axis=-1)
        for r in range(R):
            assert pick[r] in valid[r], (name, r)
    # the blocked order stays within the tighter bound of its depth
    tight = oracle.lmhead_f32_error_bound(h, w, depth=_blocked_depth(d))
    assert np.all(tight < bound)
    err = np.abs(orders["blocked16"].astype(np.float64) - z).max(axis=-1)
    assert np.all(err <= tight), (err, tight)
    _, valid_t = oracle.lmhead_valid_argmax(h, w, depth=_blocked_depth(d))
    pick = np.argmax(orders["blocked16"], axis=-1)
    assert all(pick[r] in valid_t[r] for r in range(R))


def test_near_tie_makes_both_tokens_valid():
    rng = np.random.default_rng(7)
    d = 7168
    h = _bf16(rng.standard_normal((1, d)))
    w = _bf16(rng.standard_normal((128, d)) / np.sqrt(d))
    w[40] = _bf16(3.0 * np.sign(h[0]) / np.sqrt(d))
    w[90] = w[40].copy()
    w[90, 0] = _bf16(np.array([w[40, 0] * np.float32(1.0078125)], np.float32))[0]  # one bf16 ulp larger
    z = oracle.lmhead_logits(h, w)[0]
    assert abs(z[90] - z[40]) < oracle.lmhead_f32_error_bound(h, w)[0]
    am, valid = oracle.lmhead_valid_argmax(h, w)
    assert {40, 90} <= set(int(v) for v in valid[0])


def test_bound_leaves_most_rows_decided():
    """At the Kimi hidden size the bound of a blocked evaluation still forces
    the exact token on most random rows (so a parity check stays exact almost
    everywhere); the any-order bound is far looser."""
    rng = np.random.default_rng(8)
    d, R, V = 7168, 48, 512
    h = _bf16(rng.standard_normal((R, d)))
    w = _bf16(rng.standard_normal((V, d)) / np.sqrt(d))
    _, valid = oracle.lmhead_valid_argmax(h, w, depth=_blocked_depth(d))
    assert sum(len(v) == 1 for v in valid) >= 0.9 * R
    _, loose = oracle.lmhead_valid_argmax(h, w)
    assert sum(len(v) for v in loose) > sum(len(v) for v in valid)


def test_planted_rows_take_the_planted_token():
    s = synth.custom(B=2, D=4, K=3, N=16, H=1, d_l=64, d_r=16, V=400, L=(5, 9), dtype="bf16", seed=11,
                     accept_p=0.8, accept_bias=6.0)
    x = synth.make_step(s)
    tree = oracle.build_tree(x.logp, x.tok, x.root_tok, x.cache_len, s.N)
    hidden, w, planted = synth.lmhead_inputs(s, tree["parent"], tree["node_tok"], tree["n_nodes"], d_model=64)
    hw = synth.bf16_bits_to_f32(hidden)
    ww = synth.bf16_bits_to_f32(w)
    rows = [(b, i) for b in range(2) for i in range(s.N) if planted[b, i] >= 0]
    assert len(rows) >= 4
    hit = sum(int(oracle.lmhead_argmax(hw[b, i:i + 1], ww)[0]) == planted[b, i] for b, i in rows)
    assert hit >= 0.9 * len(rows)
    # the accept walk over the head's argmax then accepts drafted nodes
    am = np.stack([oracle.lmhead_argmax(hw[b], ww) for b in range(2)])
    paths = [oracle.accept_walk(am[b], tree["node_tok"][b], tree["parent"][b], int(tree["n_nodes"][b]))
             for b in range(2)]
    assert max(len(p) for p in paths) >= 2


def test_vocab_slices_give_the_same_picks():
    """Evaluating the head one slice of the vocabulary at a time (to bound the
    widened head's memory) changes nothing: same logits, bound and valid sets."""
    rng = np.random.default_rng(8)
    h = _bf16(rng.standard_normal((7, 64)))
    w = _bf16(rng.standard_normal((1000, 64)) / 8.0)
    assert np.allclose(oracle.lmhead_logits(h, w, v_chunk=97), oracle.lmhead_logits(h, w), rtol=0, atol=1e-12)
    assert np.allclose(oracle.lmhead_f32_error_bound(h, w, 19, v_chunk=97), oracle.lmhead_f32_error_bound(h, w, 19),
                       rtol=1e-12, atol=0)
    am1, v1 = oracle.lmhead_valid_argmax(h, w, 19, v_chunk=128)
    am2, v2 = oracle.lmhead_valid_argmax(h, w, 19)
    assert np.array_equal(am1, am2) and all(np.array_equal(a, b) for a, b in zip(v1, v2))
