"""GPU parity of ddt_accept_compact_lmhead (the target's LM head folded into
the accept argmax) against the oracle's float64 head.

Every pick must be one the oracle allows for a float32 evaluation with the
rounding depth the library declares (15 + ceil(d / 16) roundings per
product); rows where the oracle allows a single token must match it exactly.
Where every row of a request is decided that way, the walk, committed tokens
and compacted cache are compared bit for bit with the oracle's accept on the
oracle's own argmax."""
import dataclasses
import math

import numpy as np
import pytest
import torch

import oracle
from ddtree_speculative_decode_b200 import lib, synth
from ddt_testutil import bf16_tensor_bits, step_to_device, t_from

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
V_CHUNK = 8192


def depth(d):
    return 15 + math.ceil(d / 16)


def _case(s, d):
    x = synth.make_step(s)
    tree = oracle.build_tree(x.logp, x.tok, x.root_tok, x.cache_len, s.N)
    hidden, w, planted = synth.lmhead_inputs(s, tree["parent"], tree["node_tok"], tree["n_nodes"], d)
    return x, tree, hidden, w, planted


def _run(s, x, tree, hidden, w, ws=None):
    d = step_to_device(x, DEV)
    kv = t_from(x.kv, DEV, True)
    cl = d["cache_len"].clone()
    out = lib.accept_compact_lmhead(t_from(hidden, DEV, True), t_from(w, DEV, True), t_from(tree["node_tok"], DEV),
                                    t_from(tree["parent"], DEV), t_from(tree["n_nodes"], DEV), kv, d["cache_off"],
                                    cl, d["cache_cap"], workspace=ws)
    torch.cuda.synchronize()
    got = {k: v.cpu().numpy() for k, v in out.items()}
    got["cache_len"] = cl.cpu().numpy()
    got["kv"] = bf16_tensor_bits(kv)
    return got


def _check(s, x, tree, hidden, w, got, reqs=None, rows_of=None):
    """Picks against the oracle's valid sets (requests `reqs`, rows
    rows_of(b) of each, default all real rows); walk and compaction of every
    fully checked request whose rows are all decided. Returns the fraction of
    decided rows."""
    d = hidden.shape[-1]
    wf = synth.bf16_bits_to_f32(w)
    reqs = range(s.B) if reqs is None else reqs
    decided = total = 0
    full = []
    for b in reqs:
        n = int(tree["n_nodes"][b])
        rows = list(range(n)) if rows_of is None else rows_of(b)
        hf = synth.bf16_bits_to_f32(hidden[b, rows])
        am, valid = oracle.lmhead_valid_argmax(hf, wf, depth(d), v_chunk=V_CHUNK)
        all_decided = True
        for j, i in enumerate(rows):
            pick = int(got["am"][b, i])
            assert pick in set(valid[j].tolist()), (b, i, pick, valid[j][:8])
            if len(valid[j]) == 1:
                decided += 1
                assert pick == int(am[j])
            else:
                all_decided = False
            total += 1
        assert np.all(got["am"][b, n:] == -1)
        if rows_of is None and all_decided:
            full.append((b, am))
    # walk + compaction on the oracle's own argmax for fully decided requests
    kv_ref = x.kv.copy()
    for b, am in full:
        onehot = np.zeros((1, s.N, s.V), np.float32)
        onehot[0, np.arange(len(am)), am] = 1.0
        sl = {k: tree[k][b:b + 1] for k in ("node_tok", "parent", "n_nodes")}
        off = int(x.cache_off[b])
        kv_b = kv_ref[off:off + int(x.cache_cap[b])]
        ref = oracle.accept_compact(onehot, "f32", sl["node_tok"], sl["parent"], sl["n_nodes"], kv_b,
                                    np.zeros(1, np.int64), x.cache_len[b:b + 1], x.cache_cap[b:b + 1])
        for k in ("acc_len", "acc_nodes", "out_tok", "bonus", "status"):
            assert np.array_equal(got[k][b:b + 1], ref[k]), (k, b)
        assert got["cache_len"][b] == ref["cache_len"][0]
        nl = int(ref["cache_len"][0])
        assert np.array_equal(got["kv"][off:off + nl], kv_b[:nl])
    return decided / max(1, total), len(full)


@pytest.mark.parametrize("B,N,D,K,d,V", [
    (2, 8, 4, 2, 64, 400),        # the pages' tiny model: hidden 64, vocabulary 400
    (3, 7, 3, 3, 200, 1000),      # ragged everywhere: rows, head width, vocabulary
    (6, 128, 16, 8, 256, 5000),   # 768 rows: two passes over the head
])
def test_lmhead_small(B, N, D, K, d, V):
    s = synth.custom(B=B, D=D, K=K, N=N, H=1, d_l=32, d_r=0, V=V, L=tuple(range(5, 5 + B)), dtype="bf16",
                     accept_p=0.8, seed=B * 1000 + d)
    x, tree, hidden, w, planted = _case(s, d)
    got = _run(s, x, tree, hidden, w)
    frac, nfull = _check(s, x, tree, hidden, w, got)
    assert frac >= 0.9 and nfull >= 1
    assert np.all(got["status"] == 0)


@pytest.fixture(scope="module")
def kimi_head():
    """The Kimi-sized head (V 163840 x d 7168, bf16, 2.35 GB) and the
    single-request workload's tree and hidden states."""
    s = synth.kimi_1req()
    return (s,) + _case(s, 7168)


def test_lmhead_kimi_one_request(kimi_head):
    """64 verify rows x the Kimi head: every row checked."""
    s, x, tree, hidden, w, planted = kimi_head
    got = _run(s, x, tree, hidden, w)
    frac, nfull = _check(s, x, tree, hidden, w, got)
    assert frac >= 0.85
    planted_rows = planted[0] >= 0
    # a planted bias dominates: those rows pick the planted token
    assert np.array_equal(got["am"][0][planted_rows], planted[0][planted_rows])


def test_lmhead_kimi_512_rows(kimi_head):
    """512 verify rows (the long-context workload's 4 x 128) against the same
    head: a full pass of two 256-row MMA parts. Request 0 is checked on every
    row (and its walk), the others on sampled rows."""
    _, _, _, _, w, _ = kimi_head
    s = dataclasses.replace(synth.kimi_4req_32k(), L=(64,) * 4)
    x = synth.make_step(s)
    tree = oracle.build_tree(x.logp, x.tok, x.root_tok, x.cache_len, s.N)
    hidden, _, _ = synth.lmhead_inputs(s, tree["parent"], tree["node_tok"], tree["n_nodes"], 7168, w_vocab=w)
    got = _run(s, x, tree, hidden, w)
    frac, nfull = _check(s, x, tree, hidden, w, got, reqs=[0])
    rng = np.random.default_rng(3)
    frac2, _ = _check(s, x, tree, hidden, w, got, reqs=[1, 2, 3],
                      rows_of=lambda b: sorted({0, 127} | set(rng.integers(0, 128, 6).tolist())))
    assert frac >= 0.85 and frac2 >= 0.7


def test_lmhead_timeout_status_is_reported():
    """A workspace whose status word holds a timeout (as a head kernel that
    gave up a wait leaves it) makes the call accept nothing: every request
    reports DDT_ERR_TIMEOUT and keeps its cache; after zeroing, the same call
    is correct."""
    s = synth.custom(B=2, D=3, K=2, N=8, H=1, d_l=32, d_r=0, V=400, L=(5, 6), dtype="bf16", seed=77, accept_p=1.0)
    x, tree, hidden, w, planted = _case(s, 64)
    ws = torch.zeros(lib.accept_compact_workspace_size(s.B, s.N, s.V), dtype=torch.uint8, device=DEV)
    ws[:4].view(torch.int32)[0] = lib.DDT_ERR_TIMEOUT
    got = _run(s, x, tree, hidden, w, ws=ws)
    assert np.all(got["status"] == lib.DDT_ERR_TIMEOUT) and np.all(got["acc_len"] == 0)
    assert np.array_equal(got["cache_len"], x.cache_len)
    assert int(ws[256:].view(torch.int64).abs().sum().item()) == 0  # the row keys were still cleared
    ws.zero_()
    got = _run(s, x, tree, hidden, w, ws=ws)
    _check(s, x, tree, hidden, w, got)
    assert np.all(got["status"] == 0)
