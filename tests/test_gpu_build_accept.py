"""GPU parity of ddt_build_tree and ddt_accept_compact against the oracle:
bit-exact tree structure, scores, masks, argmax, accepted path, committed
tokens and compacted cache rows, on the named workloads and on edge cases
(budgets 1..1024, ties, precondition violations, capacity, empty trees)."""
import numpy as np
import pytest
import torch

import oracle
from ddtree_speculative_decode_b200 import lib, synth
from ddt_testutil import check_guard, guarded, step_to_device, t_from, bf16_tensor_bits

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _tree_np(t, b=None):
    out = {k: v.cpu().numpy() for k, v in t.items()}
    out["mask"] = out["mask"].view(np.uint32)
    return out


def _compare_tree(got, ref):
    assert np.array_equal(got["n_nodes"], ref["n_nodes"])
    for k in ("node_tok", "parent", "depth", "pos", "mask"):
        assert np.array_equal(got[k], ref[k]), k
    assert np.array_equal(got["score"].view(np.uint32), ref["score"].view(np.uint32)), "score bits"
    assert np.array_equal(got["status"], ref["status"])


def _run_build(x: synth.StepInputs, N: int):
    d = step_to_device(x, DEV)
    B = x.logp.shape[0]
    W = (N + 31) // 32
    out = lib.alloc_tree(B, N, DEV)
    bufs = {}
    for k, shape, dt, fill in (("node_tok", (B, N), torch.int32, -777), ("mask", (B, N, W), torch.int32, -777),
                                ("score", (B, N), torch.float32, 1234.5), ("n_nodes", (B,), torch.int32, -777)):
        out[k], bufs[k] = guarded(shape, dt, DEV, fill)
    lib.build_tree(d["logp"], d["tok"], d["root_tok"], d["cache_len"], N, out=out)
    torch.cuda.synchronize()
    for k, (shape, fill) in {"node_tok": ((B, N), -777), "mask": ((B, N, W), -777), "score": ((B, N), 1234.5),
                             "n_nodes": ((B,), -777)}.items():
        check_guard(bufs[k], int(np.prod(shape)), fill)
    return _tree_np(out)


@pytest.mark.parametrize("name", ["tiny-f32", "kimi-1req", "kimi-16req", "kimi-4req-32k"])
def test_build_named(name):
    s = synth.NAMED[name]()
    x = synth.make_step(s)
    got = _run_build(x, s.N)
    ref = oracle.build_tree(x.logp, x.tok, x.root_tok, x.cache_len, s.N)
    _compare_tree(got, ref)


# Covers every kernel variant: rank tuples that fit a 25-bit field (bits per
# level x min(D, N) <= 25) with N <= 64 / 128 / 256, wider tuples with the same
# three budgets, and N > 256 (shared-memory frontier); 25 and 28 bits sit on
# either side of the packed-key limit.
EDGE = [(1, 1, 1), (3, 2, 2), (4, 3, 31), (4, 3, 32), (4, 3, 33), (8, 8, 255), (8, 8, 256), (8, 16, 1024),
        (16, 8, 128), (5, 1, 40), (2, 32, 700), (64, 2, 64), (12, 31, 300), (8, 8, 100), (16, 8, 200),
        (5, 32, 64), (7, 16, 64), (25, 2, 26), (26, 2, 27)]


@pytest.mark.parametrize("D,K,N", EDGE)
@pytest.mark.parametrize("quant", [None, 0.5])
def test_build_edges(D, K, N, quant):
    rng = np.random.default_rng(D * 7919 + K * 31 + N)
    B = 5
    x = -np.abs(rng.standard_normal((B, D, K))) * 3
    if quant:
        x = -np.round(-x / quant) * quant
    logp = (-np.sort(-x, axis=2)).astype(np.float32)
    tok = rng.integers(0, 163840, size=(B, D, K)).astype(np.int32)
    root = rng.integers(0, 100, size=B).astype(np.int32)
    L = rng.integers(0, 5000, size=B).astype(np.int32)
    d = {k: t_from(v, DEV) for k, v in (("logp", logp), ("tok", tok), ("root", root), ("L", L))}
    out = lib.build_tree(d["logp"], d["tok"], d["root"], d["L"], N)
    torch.cuda.synchronize()
    _compare_tree(_tree_np(out), oracle.build_tree(logp, tok, root, L, N))


@pytest.mark.parametrize("bad", ["nan", "pos", "unsorted", "ninf"])
def test_build_precondition_status(bad):
    logp = np.array([[[-0.1, -0.5], [-0.2, -0.9]], [[-0.1, -0.5], [-0.2, -0.9]]], np.float32)
    v = {"nan": np.nan, "pos": 0.5, "ninf": -np.inf}.get(bad)
    if bad == "unsorted":
        logp[1, 1] = [-0.9, -0.2]
    else:
        logp[1, 0, 1] = v
    tok = np.arange(8, dtype=np.int32).reshape(2, 2, 2)
    root, L = np.array([5, 6], np.int32), np.array([3, 4], np.int32)
    out = lib.build_tree(t_from(logp, DEV), t_from(tok, DEV), t_from(root, DEV), t_from(L, DEV), 6)
    torch.cuda.synchronize()
    got = _tree_np(out)
    ref = oracle.build_tree(logp, tok, root, L, 6)
    _compare_tree(got, ref)
    assert got["status"][1] == lib.DDT_ERR_INPUT and got["n_nodes"][1] == 0 and got["status"][0] == 0


def test_build_host_validation():
    z = torch.zeros(1, 2, 2, device=DEV)
    zi = torch.zeros(1, 2, 2, dtype=torch.int32, device=DEV)
    o = torch.zeros(1, dtype=torch.int32, device=DEV)
    with pytest.raises(lib.DDTError) as e:
        lib.build_tree(z, zi, o, o, 2000)
    assert e.value.status == lib.DDT_ERR_INVALID_ARG


# ---------------------------------------------------------------------------
# accept + compaction
# ---------------------------------------------------------------------------


def _accept_case(s: synth.Shape, n_layers=1):
    x = synth.make_step(s)
    tree = oracle.build_tree(x.logp, x.tok, x.root_tok, x.cache_len, s.N)
    logits = synth.target_logits(s, tree["parent"], tree["node_tok"], tree["n_nodes"])
    return x, tree, logits


def _run_accept_and_compare(s, x, tree, logits, n_layers=1, stride=0, kv_host=None):
    bf = s.dtype == "bf16"
    d = step_to_device(x, DEV)
    kv_np = x.kv if kv_host is None else kv_host
    kv = t_from(kv_np, DEV, bf)
    lg = t_from(logits, DEV, bf)
    cl = d["cache_len"].clone()
    out = lib.accept_compact(lg, t_from(tree["node_tok"], DEV), t_from(tree["parent"], DEV),
                             t_from(tree["n_nodes"], DEV), kv, d["cache_off"], cl, d["cache_cap"],
                             n_layers=n_layers, layer_stride_rows=stride)
    torch.cuda.synchronize()
    kv_ref = kv_np.copy()
    ref = oracle.accept_compact(logits, s.dtype, tree["node_tok"], tree["parent"], tree["n_nodes"], kv_ref,
                                x.cache_off, x.cache_len, x.cache_cap, n_layers=n_layers, layer_stride_rows=stride)
    got = {k: v.cpu().numpy() for k, v in out.items()}
    for k in ("am", "acc_len", "acc_nodes", "out_tok", "bonus", "status"):
        assert np.array_equal(got[k], ref[k]), k
    assert np.array_equal(cl.cpu().numpy(), ref["cache_len"])
    kv_got = bf16_tensor_bits(kv) if bf else kv.cpu().numpy()
    # committed rows [0, new cache_len) of every request must match bit for bit
    for layer in range(n_layers):
        for b in range(len(x.cache_len)):
            o = int(x.cache_off[b]) + layer * stride
            nl = int(ref["cache_len"][b])
            assert np.array_equal(kv_got[o:o + nl], kv_ref[o:o + nl]), (layer, b)
    return got, ref


@pytest.mark.parametrize("name", ["tiny-f32", "kimi-1req", "kimi-16req", "kimi-4req-32k"])
def test_accept_named(name):
    s = synth.NAMED[name]()
    x, tree, logits = _accept_case(s)
    got, ref = _run_accept_and_compare(s, x, tree, logits)
    if s.B > 1:
        assert got["acc_len"].sum() > 0  # the bias makes some drafts acceptable


@pytest.mark.parametrize("V", [1, 7, 8, 9, 16383, 16384, 16385, 40000])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_accept_vocab_edges(V, dtype):
    s = synth.custom(B=3, D=3, K=3, N=12, H=1, d_l=16, d_r=8, V=V, L=(0, 5, 33), dtype=dtype, seed=V,
                     accept_p=0.9)
    x, tree, logits = _accept_case(s)
    _run_accept_and_compare(s, x, tree, logits)


def test_accept_ties_and_multilayer():
    s = synth.custom(B=2, D=4, K=2, N=10, H=1, d_l=32, d_r=0, V=300, L=(4, 9), dtype="bf16", seed=9,
                     accept_p=1.0)
    x, tree, logits = _accept_case(s)
    # force ties: duplicate each row's max at a higher index
    for b in range(2):
        for i in range(10):
            m = np.argmax(synth.bf16_bits_to_f32(logits[b, i]))
            logits[b, i, (m + 17) % 300] = logits[b, i, m]
    # two layers: the pool repeated at a stride
    rows = x.kv.shape[0]
    stride = rows + 5
    kv2 = np.zeros((stride * 2, x.kv.shape[1]), x.kv.dtype)
    kv2[:rows] = x.kv
    kv2[stride:stride + rows] = x.kv[::-1]
    _run_accept_and_compare(s, x, tree, logits, n_layers=2, stride=stride, kv_host=kv2)


def test_accept_many_layers():
    """61 layers (the Kimi model's depth) at a stride, each holding different
    rows: every layer compacted along the same accepted path."""
    s = synth.custom(B=3, D=4, K=3, N=16, H=1, d_l=64, d_r=16, V=500, L=(7, 0, 40), dtype="bf16", seed=61,
                     accept_p=0.9)
    x, tree, logits = _accept_case(s)
    rows, n_layers = x.kv.shape[0], 61
    stride = rows + 3
    kvl = np.zeros((stride * n_layers, x.kv.shape[1]), x.kv.dtype)
    for layer in range(n_layers):
        kvl[layer * stride:layer * stride + rows] = np.roll(x.kv, layer, axis=0)
    got, _ = _run_accept_and_compare(s, x, tree, logits, n_layers=n_layers, stride=stride, kv_host=kvl)
    assert got["acc_len"].sum() > 0


def test_accept_capacity_and_empty_tree():
    s = synth.custom(B=3, D=3, K=2, N=6, H=1, d_l=8, d_r=0, V=50, L=(3, 3, 3), seed=4)
    x, tree, logits = _accept_case(s)
    x.cache_cap[1] = 3 + 2  # too small for 6 tree rows
    tree["n_nodes"][2] = 0
    got, ref = _run_accept_and_compare(s, x, tree, logits)
    assert got["status"][1] == lib.DDT_ERR_CAPACITY and got["acc_len"][1] == 0 and got["bonus"][1] == -1
    assert got["bonus"][2] == -1 and got["status"][2] == 0
