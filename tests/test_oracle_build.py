"""Pins for the oracle's best-first tree build, against things other than
itself: brute-force enumerate-and-sort of every rank path on tiny inputs (ties
forced by quantised log-probs), the oracle-drafter chain the capstone page
describes, the K = 1 chain, and the degenerate budgets."""
import itertools

import numpy as np
import pytest

from oracle import build_tree, ERR_INPUT
from ddtree_speculative_decode_b200 import synth


def _sorted_logp(rng, D, K, quant=None):
    x = -np.abs(rng.standard_normal((D, K))) * 2.0
    if quant:
        x = -np.round(-x / quant) * quant
    x = -np.sort(-x, axis=1)  # descending
    return x.astype(np.float32)


def brute_force_tree(logp, tok, root, L, N):
    """Enumerate every rank path, score it left to right in float32, sort by
    (score desc, depth asc, ranks lexicographic asc), keep the first N - 1."""
    D, K = logp.shape
    paths = []
    for d in range(1, D + 1):
        for ranks in itertools.product(range(K), repeat=d):
            s = np.float32(0.0)
            for j, r in enumerate(ranks):
                s = np.float32(s + logp[j, r])
            paths.append((-float(s), d, ranks, s))
    paths.sort(key=lambda t: (t[0], t[1], t[2]))
    chosen = [p[2] for p in paths[:N - 1]]
    n = 1 + len(chosen)
    idx = {(): 0}
    for i, r in enumerate(chosen, start=1):
        idx[r] = i
    W = (N + 31) // 32
    node_tok = np.full(N, -1, np.int32)
    parent = np.full(N, -1, np.int32)
    depth = np.full(N, -1, np.int32)
    pos = np.full(N, -1, np.int32)
    score = np.full(N, -np.inf, np.float32)
    mask = np.zeros((N, W), np.uint32)
    node_tok[0], depth[0], pos[0], score[0] = root, 0, L, 0.0
    for i, r in enumerate(chosen, start=1):
        node_tok[i] = tok[len(r) - 1, r[-1]]
        parent[i] = idx[r[:-1]]
        depth[i] = len(r)
        pos[i] = L + len(r)
        s = np.float32(0.0)
        for j, rr in enumerate(r):
            s = np.float32(s + logp[j, rr])
        score[i] = s
    # ancestor sets from the prefix relation, not from parent pointers
    all_paths = [()] + chosen
    for i, r in enumerate(all_paths):
        for j, a in enumerate(all_paths):
            if len(a) <= len(r) and r[:len(a)] == a:
                mask[i, j >> 5] |= np.uint32(1 << (j & 31))
    return dict(node_tok=node_tok, parent=parent, depth=depth, pos=pos, score=score, mask=mask, n_nodes=n)


CASES = [(D, K, N, q) for D in (1, 2, 3, 4) for K in (1, 2, 3) for N in (1, 2, 5, 9, 40, 70)
         for q in (None, 0.5)]


@pytest.mark.parametrize("D,K,N,quant", CASES)
def test_build_equals_brute_force(D, K, N, quant):
    rng = np.random.default_rng(D * 1000 + K * 100 + N + (7 if quant else 0))
    B = 2
    logp = np.stack([_sorted_logp(rng, D, K, quant) for _ in range(B)])
    tok = rng.integers(0, 1000, size=(B, D, K)).astype(np.int32)
    root = np.array([11, 22], np.int32)
    L = np.array([5, 0], np.int32)
    got = build_tree(logp, tok, root, L, N)
    for b in range(B):
        ref = brute_force_tree(logp[b], tok[b], root[b], L[b], N)
        assert got["n_nodes"][b] == ref["n_nodes"]
        for k in ("node_tok", "parent", "depth", "pos", "mask"):
            np.testing.assert_array_equal(got[k][b], ref[k], err_msg=k)
        np.testing.assert_array_equal(got["score"][b].view(np.uint32), ref["score"].view(np.uint32))


def test_ties_are_exercised():
    # with quantised log-probs equal scores across different paths do occur
    rng = np.random.default_rng(5)
    logp = _sorted_logp(rng, 4, 3, 0.5)
    scores = []
    for d in range(1, 5):
        for r in itertools.product(range(3), repeat=d):
            scores.append(float(sum(logp[j, x] for j, x in enumerate(r))))
    assert len(scores) > len(set(scores))


def test_oracle_drafter_gives_chain():
    # rank-0 log-prob 0 at every depth: the golden continuation is popped first
    golden = np.array([5, 9, 3, 7, 1, 2, 8], np.int32)
    for D, N in ((7, 8), (4, 8), (7, 4), (7, 20)):
        lp, tk = synth.oracle_drafter(golden, D, 3)
        t = build_tree(lp[None], tk[None], np.array([42]), np.array([10]), N)
        chain = min(D, N - 1)
        for i in range(1, chain + 1):
            assert t["depth"][0, i] == i
            assert t["parent"][0, i] == i - 1
            assert t["node_tok"][0, i] == golden[i - 1]
            assert t["score"][0, i] == 0.0
        assert t["n_nodes"][0] == min(N, 1 + sum(3 ** d for d in range(1, D + 1)))


def test_topk1_is_chain():
    rng = np.random.default_rng(3)
    lp = -np.abs(rng.standard_normal((1, 6, 1))).astype(np.float32)
    tk = np.arange(6, dtype=np.int32).reshape(1, 6, 1)
    t = build_tree(lp, tk, np.array([0]), np.array([3]), 32)
    assert t["n_nodes"][0] == 7
    np.testing.assert_array_equal(t["parent"][0, :7], [-1, 0, 1, 2, 3, 4, 5])
    np.testing.assert_array_equal(t["pos"][0, :7], 3 + np.arange(7))
    # chain masks are prefix masks
    np.testing.assert_array_equal(t["mask"][0, :7, 0], [(1 << (i + 1)) - 1 for i in range(7)])


def test_budget_one_is_root_only():
    lp = np.full((1, 3, 2), -1.0, np.float32)
    t = build_tree(lp, np.zeros((1, 3, 2), np.int32), np.array([77]), np.array([4]), 1)
    assert t["n_nodes"][0] == 1 and t["node_tok"][0, 0] == 77 and t["mask"][0, 0, 0] == 1


def test_mask_word_layout_past_32_nodes():
    rng = np.random.default_rng(11)
    lp = _sorted_logp(rng, 3, 4, None)[None]
    t = build_tree(lp, np.zeros((1, 3, 4), np.int32), np.array([0]), np.array([0]), 70)
    assert t["n_nodes"][0] == 70 and t["mask"].shape == (1, 70, 3)
    for i in (33, 64, 69):
        assert (t["mask"][0, i, i >> 5] >> np.uint32(i & 31)) & 1
        assert t["mask"][0, i, 0] & 1  # root always visible


@pytest.mark.parametrize("bad", ["nan", "pos", "unsorted", "inf"])
def test_precondition_violation(bad):
    lp = np.array([[[-0.1, -0.5], [-0.2, -0.9]]], np.float32)
    if bad == "nan":
        lp[0, 1, 1] = np.nan
    elif bad == "pos":
        lp[0, 0, 0] = 0.25
    elif bad == "unsorted":
        lp[0, 1] = [-0.9, -0.2]
    else:
        lp[0, 0, 1] = -np.inf
    t = build_tree(lp, np.zeros((1, 2, 2), np.int32), np.array([1]), np.array([2]), 4)
    assert t["status"][0] == ERR_INPUT and t["n_nodes"][0] == 0
    assert np.all(t["node_tok"][0] == -1) and np.all(t["mask"][0] == 0)


def _key(score, ranks):
    # the build's total order: score descending, depth ascending, ranks lexicographic
    return (-float(score), len(ranks), tuple(ranks))


@pytest.mark.parametrize("D,K,N,quant", [(64, 32, 1024, None), (64, 32, 1024, 0.5), (8, 8, 64, 0.25),
                                         (16, 8, 128, None), (6, 6, 32, 0.5), (3, 32, 700, 0.5),
                                         (64, 1, 1024, None), (64, 2, 1024, 0.5), (12, 16, 256, 1.0)])
def test_build_is_the_best_prefix_closed_set_at_full_sizes(D, K, N, quant):
    """Where enumerating K^D paths is out of reach: the tree is prefix-closed,
    its scores are the left-to-right float32 sums, its nodes come in the
    order's sequence, and every unselected child of a selected path orders
    after the last selected one. Since log-probs are <= 0, any unselected
    path orders no earlier than its first unselected prefix, which is such a
    child; so the tree holds exactly the N - 1 best paths."""
    rng = np.random.default_rng(D * 1000 + K * 10 + N)
    logp = _sorted_logp(rng, D, K, quant)
    tok = np.stack([rng.permutation(50000)[:K] for _ in range(D)]).astype(np.int32)
    t = build_tree(logp[None], tok[None], np.array([7]), np.array([100]), N)
    n = int(t["n_nodes"][0])
    total = sum(K ** d for d in range(1, D + 1))  # exact integers
    assert n - 1 == min(N - 1, total)
    rank_of = [{int(tok[d, r]): r for r in range(K)} for d in range(D)]
    ranks = [()]
    score = [np.float32(0.0)]
    for i in range(1, n):
        p = int(t["parent"][0, i])
        d = int(t["depth"][0, i])
        assert 0 <= p < i and d == len(ranks[p]) + 1 and d <= D
        r = rank_of[d - 1][int(t["node_tok"][0, i])]
        ranks.append(ranks[p] + (r,))
        score.append(np.float32(score[p] + logp[d - 1, r]))
        assert np.float32(t["score"][0, i]).view(np.uint32) == score[i].view(np.uint32)
        assert int(t["pos"][0, i]) == 100 + d
    keys = [_key(score[i], ranks[i]) for i in range(1, n)]
    assert all(a < b for a, b in zip(keys, keys[1:]))
    chosen = set(ranks)
    last = keys[-1] if keys else None
    for i in range(n):
        if len(ranks[i]) == D:
            continue
        for r in range(K):
            c = ranks[i] + (r,)
            if c not in chosen:
                s = np.float32(score[i] + logp[len(ranks[i]), r])
                assert _key(s, c) > last, (c, last)
    # masks: ancestors by the prefix relation
    idx = {rk: i for i, rk in enumerate(ranks)}
    for i in range(n):
        want = {idx[ranks[i][:j]] for j in range(len(ranks[i]) + 1)}
        got = {j for j in range(n) if (int(t["mask"][0, i, j >> 5]) >> (j & 31)) & 1}
        assert got == want
