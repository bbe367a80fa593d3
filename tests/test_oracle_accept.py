"""Pins for the oracle's greedy accept walk and latent-KV compaction: the
oracle-drafter loop statistics the pages print (tests/golden), the all-reject
case, brute force over every root-to-node path, and a non-contiguous accepted
path whose compaction must read every source row before writing."""
import os

import numpy as np
import pytest

from oracle import accept_compact, accept_walk, build_tree, ERR_CAPACITY
from ddtree_speculative_decode_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "capstone_ddtree_stats.txt")


def _read_golden():
    vals = {}
    for line in open(GOLDEN):
        line = line.strip()
        if line and not line.startswith("#"):
            k, v = line.split()
            vals[k] = v
    return vals


def _toy_target(ctx, V):
    """A deterministic stand-in for the target model's greedy choice."""
    h = 0
    for i, t in enumerate(ctx[-4:]):
        h = (h * 1000003 + (i + 1) * (int(t) + 17)) & 0xFFFFFFFF
    return (h * 2654435761 + len(ctx)) % V


def _one_hot_logits(rows_ctx, N, V):
    lg = np.zeros((1, N, V), np.float32)
    for i, ctx in enumerate(rows_ctx):
        lg[0, i, _toy_target(ctx, V)] = 1.0
    return lg


def test_pages_loop_statistics():
    """Oracle drafter + greedy target: DDTree equals AR token for token, with
    the step / accept counts the capstone page reports."""
    g = _read_golden()
    T, blk, budget = int(g["tokens"]), int(g["block_size"]), int(g["budget"])
    assert budget == blk - 1
    V, K = 400, 3
    prompt = [3, 14, 15, 92, 65]
    # autoregressive reference: one target forward per token
    ctx, ar = list(prompt), []
    for _ in range(T):
        ar.append(_toy_target(ctx, V))
        ctx.append(ar[-1])
    ar_forwards = T
    # DDTree: the prefill yields the first token (the first root)
    committed = [_toy_target(prompt, V)]
    L = len(prompt)
    pool = np.zeros((L + 64 * blk, 1), np.float32)
    pool[:L, 0] = prompt
    steps = 0
    while len(committed) < T:
        lp, tk = synth.oracle_drafter(np.array(ar[len(committed):], np.int32), budget, K,
                                      sentinel_from=T - len(committed))
        t = build_tree(lp[None], tk[None], np.array([committed[-1]]), np.array([L]), blk)
        n = int(t["n_nodes"][0])
        # each tree row's latent KV stands in as its token id
        pool[L:L + n, 0] = t["node_tok"][0, :n]
        rows_ctx = []
        for i in range(n):
            path, j = [], i
            while j >= 0:
                path.append(int(t["node_tok"][0, j]))
                j = int(t["parent"][0, j])
            rows_ctx.append(prompt + committed[:-1] + path[::-1])
        lg = _one_hot_logits(rows_ctx, blk, V)
        r = accept_compact(lg, "f32", t["node_tok"], t["parent"], t["n_nodes"], pool, np.array([0]),
                           np.array([L], np.int32), np.array([len(pool)], np.int32))
        a = int(r["acc_len"][0])
        committed += [int(x) for x in r["out_tok"][0, :a + 1]]
        L = int(r["cache_len"][0])
        steps += 1
    assert committed[:T] == ar
    assert steps == int(g["steps"]) == int(g["target_forwards_ddtree"])
    assert len(committed) == int(g["committed"])
    assert ar_forwards == int(g["target_forwards_ar"])
    assert "%.2f" % ((len(committed) - 1) / steps) == g["avg_accept"]
    # the compacted cache holds the prompt followed by every committed token but the last root
    np.testing.assert_array_equal(pool[:L, 0], prompt + committed[:-1])


def test_all_reject():
    s = synth.custom(B=1, D=3, K=2, N=6, H=1, d_l=4, d_r=0, V=30, L=(4,), seed=1)
    x = synth.make_step(s)
    t = build_tree(x.logp, x.tok, x.root_tok, x.cache_len, s.N)
    lg = np.zeros((1, s.N, s.V), np.float32)
    used = set(int(v) for v in t["node_tok"][0])
    miss = [v for v in range(s.V) if v not in used][0]
    lg[0, :, miss] = 1.0
    kv = x.kv.copy()
    r = accept_compact(lg, "f32", t["node_tok"], t["parent"], t["n_nodes"], kv, x.cache_off, x.cache_len,
                       x.cache_cap)
    assert r["acc_len"][0] == 0 and r["bonus"][0] == miss
    assert list(r["out_tok"][0, :1]) == [miss] and r["cache_len"][0] == 5
    np.testing.assert_array_equal(kv, x.kv)  # root row copied onto itself


def _all_paths(parent, n):
    paths = []
    for i in range(n):
        p, j = [], i
        while j >= 0:
            p.append(j)
            j = int(parent[j])
        paths.append(p[::-1])
    return paths


@pytest.mark.parametrize("seed", range(12))
def test_walk_equals_brute_force(seed):
    s = synth.custom(B=3, D=4, K=3, N=20, H=1, d_l=4, d_r=0, V=40, L=(2, 9, 0), seed=100 + seed,
                     accept_p=0.8)
    x = synth.make_step(s)
    t = build_tree(x.logp, x.tok, x.root_tok, x.cache_len, s.N)
    lg = synth.target_logits(s, t["parent"], t["node_tok"], t["n_nodes"])
    kv = x.kv.copy()
    r = accept_compact(lg, "f32", t["node_tok"], t["parent"], t["n_nodes"], kv, x.cache_off, x.cache_len,
                       x.cache_cap)
    for b in range(s.B):
        n = int(t["n_nodes"][b])
        am = lg[b, :n].argmax(-1)
        # valid paths: every step's token is the target's greedy choice at its parent
        best = [0]
        for p in _all_paths(t["parent"][b], n):
            if all(t["node_tok"][b, p[k]] == am[p[k - 1]] for k in range(1, len(p))) and len(p) > len(best):
                best = p
        a = len(best) - 1
        assert r["acc_len"][b] == a
        np.testing.assert_array_equal(r["acc_nodes"][b, :a + 1], best)
        assert r["bonus"][b] == am[best[-1]]
        off, L = int(x.cache_off[b]), int(x.cache_len[b])
        np.testing.assert_array_equal(kv[off:off + L], x.kv[off:off + L])
        for j, p in enumerate(best):
            np.testing.assert_array_equal(kv[off + L + j], x.kv[off + L + p])


def test_noncontiguous_path_reads_before_writes():
    # tree: 0 -> 2 -> 3 -> 5 accepted; 1, 4 rejected siblings
    parent = np.array([[-1, 0, 0, 2, 2, 3]], np.int32)
    node_tok = np.array([[9, 10, 11, 12, 13, 14]], np.int32)
    V = 20
    lg = np.zeros((1, 6, V), np.float32)
    lg[0, 0, 11] = 1  # root -> node 2
    lg[0, 2, 12] = 1  # node 2 -> node 3
    lg[0, 3, 14] = 1  # node 3 -> node 5
    lg[0, 5, 7] = 1  # bonus
    lg[0, 1, 0] = lg[0, 4, 0] = 1
    L = 3
    kv = np.arange((L + 6) * 2, dtype=np.float32).reshape(L + 6, 2)
    before = kv.copy()
    r = accept_compact(lg, "f32", node_tok, parent, np.array([6]), kv, np.array([0]), np.array([L]),
                       np.array([L + 6]))
    assert list(r["acc_nodes"][0, :4]) == [0, 2, 3, 5] and r["acc_len"][0] == 3
    assert list(r["out_tok"][0, :4]) == [11, 12, 14, 7]
    # naive in-order copy without reading first would also pass here because
    # path[j] >= j; a second layer checks the layer stride
    for j, p in enumerate([0, 2, 3, 5]):
        np.testing.assert_array_equal(kv[L + j], before[L + p])
    np.testing.assert_array_equal(kv[:L], before[:L])


def test_multi_layer_and_capacity():
    parent = np.array([[-1, 0, 1], [-1, 0, 1]], np.int32)
    node_tok = np.array([[5, 6, 7], [5, 6, 7]], np.int32)
    lg = np.zeros((2, 3, 10), np.float32)
    lg[:, 0, 6] = 1
    lg[:, 1, 7] = 1
    lg[:, 2, 1] = 1
    stride = 20
    kv = np.arange(2 * stride, dtype=np.float32).reshape(2 * stride, 1)
    before = kv.copy()
    # request 0 fits (L 2 + 3 <= cap 5); request 1 does not (cap 4)
    r = accept_compact(lg, "f32", node_tok, parent, np.array([3, 3]), kv, np.array([0, 8]), np.array([2, 2]),
                       np.array([5, 4]), n_layers=2, layer_stride_rows=stride)
    assert r["acc_len"][0] == 2 and r["cache_len"][0] == 5
    assert r["status"][1] == ERR_CAPACITY and r["cache_len"][1] == 2
    np.testing.assert_array_equal(kv, before)  # chain path 0,1,2 copies in place
    # a non-trivial two-layer copy
    lg2 = np.zeros((1, 3, 10), np.float32)
    lg2[0, 0, 7] = 1
    parent2 = np.array([[-1, 0, 0]], np.int32)
    kv2 = before.copy()
    r2 = accept_compact(lg2, "f32", node_tok[:1], parent2, np.array([3]), kv2, np.array([0]), np.array([2]),
                        np.array([5]), n_layers=2, layer_stride_rows=stride)
    assert list(r2["acc_nodes"][0, :2]) == [0, 2]
    for layer in range(2):
        np.testing.assert_array_equal(kv2[layer * stride + 3], before[layer * stride + 4])


def test_many_layers_equal_one_layer_each():
    """61 layers at a stride are 61 independent copies along the same path:
    each layer's slice ends as a one-layer call on that slice alone leaves it,
    and the gap rows between layers stay untouched."""
    rng = np.random.default_rng(61)
    parent = np.array([[-1, 0, 0, 1, 2, 4, 4]], np.int32)
    node_tok = np.array([[9, 3, 4, 5, 6, 7, 8]], np.int32)
    lg = rng.standard_normal((1, 7, 12)).astype(np.float32)
    lg[0, 0, 4] = 9.0  # root -> node 2
    lg[0, 2, 6] = 9.0  # node 2 -> node 4
    lg[0, 4, 8] = 9.0  # node 4 -> node 6
    L, n_layers, rows = 5, 61, 12
    stride = rows + 2
    kv = rng.standard_normal((n_layers * stride, 3))
    before = kv.copy()
    r = accept_compact(lg, "f32", node_tok, parent, np.array([7]), kv, np.array([0]), np.array([L]),
                       np.array([L + 7]), n_layers=n_layers, layer_stride_rows=stride)
    assert list(r["acc_nodes"][0, :4]) == [0, 2, 4, 6] and r["acc_len"][0] == 3
    for layer in range(n_layers):
        one = before[layer * stride:layer * stride + rows].copy()
        r1 = accept_compact(lg, "f32", node_tok, parent, np.array([7]), one, np.array([0]), np.array([L]),
                            np.array([L + 7]))
        assert r1["acc_len"][0] == 3
        np.testing.assert_array_equal(kv[layer * stride:layer * stride + rows], one)
        np.testing.assert_array_equal(kv[layer * stride + rows:(layer + 1) * stride],
                                      before[layer * stride + rows:(layer + 1) * stride])
        for j, node in enumerate([0, 2, 4, 6]):
            np.testing.assert_array_equal(kv[layer * stride + L + j], before[layer * stride + L + node])


def test_walk_picks_lowest_index_on_duplicate_tokens():
    parent = [-1, 0, 0]
    node_tok = [1, 5, 5]
    assert accept_walk([5, 0, 0], node_tok, parent, 3) == [0, 1]


def test_argmax_ties_take_lowest_index_bf16():
    from oracle import row_argmax, widen_logits
    x = np.zeros((2, 9), np.float32)
    x[0, [3, 7]] = 2.5
    x[1, [0, 8]] = -0.5
    x[1, 1:8] = -1.0
    bits = synth.f32_to_bf16_bits(x)
    assert list(row_argmax(widen_logits(bits, "bf16"))) == [3, 0]
