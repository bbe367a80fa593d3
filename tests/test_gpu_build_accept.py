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
# three budgets (N 129..256 with D <= 16 and K <= 16: the level-synchronous
# build), and N > 256 (shared-memory frontier); 25 and 28 bits sit on either
# side of the packed-key limit.
EDGE = [(1, 1, 1), (3, 2, 2), (4, 3, 31), (4, 3, 32), (4, 3, 33), (8, 8, 255), (8, 8, 256), (8, 16, 1024),
        (16, 8, 128), (5, 1, 40), (2, 32, 700), (64, 2, 64), (12, 31, 300), (8, 8, 100), (16, 8, 200),
        (5, 32, 64), (7, 16, 64), (25, 2, 26), (26, 2, 27), (8, 16, 256), (7, 16, 129), (16, 16, 256),
        (7, 13, 250), (20, 8, 256)]


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
    """The workloads' own seeded logits. Whatever they accept must match the
    oracle; the single-request draw happens to reject at the root (its biased
    child scores below the row's N(0, 1) maximum), so acceptance of long paths
    is checked separately with planted logits below."""
    s = synth.NAMED[name]()
    x, tree, logits = _accept_case(s)
    _run_accept_and_compare(s, x, tree, logits)


def _set_logit(logits, dtype, b, i, v, value):
    if dtype == "bf16":
        logits[b, i, v] = synth.f32_to_bf16_bits(np.array([value], np.float32))[0]
    else:
        logits[b, i, v] = value


def _deepest_path(tree, b):
    n = int(tree["n_nodes"][b])
    node = int(np.argmax(tree["depth"][b, :n]))  # deepest node, lowest index on ties
    path = []
    while node > 0:
        path.append(node)
        node = int(tree["parent"][b, node])
    return path[::-1]


@pytest.mark.parametrize("name", ["tiny-f32", "kimi-1req", "kimi-16req", "kimi-4req-32k"])
def test_accept_planted_deepest_path(name):
    """Along each tree's deepest path the next node's token is made the row's
    argmax, so every request accepts that whole path (several tokens per step,
    as the pages' runs do) and the compaction moves a long, non-contiguous set
    of rows."""
    s = synth.NAMED[name]()
    x, tree, logits = _accept_case(s)
    want = []
    for b in range(s.B):
        path = _deepest_path(tree, b)
        prev = 0
        for node in path:
            _set_logit(logits, s.dtype, b, prev, int(tree["node_tok"][b, node]), 30.0)
            prev = node
        want.append(len(path))
    got, ref = _run_accept_and_compare(s, x, tree, logits)
    assert np.array_equal(got["acc_len"], np.array(want, np.int32))
    # every request accepts several drafts (how many depends on the tree: the
    # workloads' drafters spread their mass over many tokens, so the budget
    # goes to siblings and the trees are 2 to 3 nodes deep)
    assert min(want) >= 2


@pytest.mark.parametrize("name", ["tiny-f32", "kimi-1req", "kimi-16req"])
def test_accept_reject_path(name):
    """Every child's token is pushed far below its parent row's maximum: no
    draft is accepted, the bonus is the root row's argmax and only the root's
    row is committed."""
    s = synth.NAMED[name]()
    x, tree, logits = _accept_case(s)
    for b in range(s.B):
        n = int(tree["n_nodes"][b])
        for c in range(1, n):
            _set_logit(logits, s.dtype, b, int(tree["parent"][b, c]), int(tree["node_tok"][b, c]), -30.0)
    got, ref = _run_accept_and_compare(s, x, tree, logits)
    assert np.all(got["acc_len"] == 0)
    assert np.array_equal(got["bonus"], got["am"][:, 0])
    assert np.array_equal(got["acc_nodes"][:, 0], np.zeros(s.B, np.int32))


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


def test_accept_node_count_and_pool_bounds():
    """Device-side guards: a request whose n_nodes exceeds N is bad input, and
    one whose compaction rows would fall outside the pool is out of bounds;
    both are skipped (nothing copied, cache_len kept) while the others match
    the oracle."""
    s = synth.custom(B=4, D=3, K=3, N=10, H=1, d_l=32, d_r=8, V=700, L=(5, 9, 2, 4), dtype="bf16", seed=3,
                     accept_p=1.0)
    x, tree, logits = _accept_case(s)
    d = step_to_device(x, DEV)
    kv = t_from(x.kv, DEV, True)
    rows = x.kv.shape[0]
    off = x.cache_off.copy()
    off[1] = rows - 3               # rows [off + L, off + L + n) run past the pool
    nn = tree["n_nodes"].copy()
    nn[2] = s.N + 1                 # more nodes than rows per request
    cl = d["cache_len"].clone()
    out = lib.accept_compact(t_from(logits, DEV, True), t_from(tree["node_tok"], DEV), t_from(tree["parent"], DEV),
                             t_from(nn, DEV), kv, t_from(off, DEV), cl, d["cache_cap"])
    torch.cuda.synchronize()
    got = {k: v.cpu().numpy() for k, v in out.items()}
    assert got["status"][1] == lib.DDT_ERR_BOUNDS and got["status"][2] == lib.DDT_ERR_INPUT
    for b in (1, 2):
        assert got["acc_len"][b] == 0 and got["bonus"][b] == -1
        assert np.all(got["acc_nodes"][b] == -1) and np.all(got["out_tok"][b] == -1)
    assert np.array_equal(cl.cpu().numpy()[[1, 2]], x.cache_len[[1, 2]])
    kv_ref = x.kv.copy()
    keep = tree["n_nodes"].copy()
    keep[[1, 2]] = 0
    ref = oracle.accept_compact(logits, "bf16", tree["node_tok"], tree["parent"], keep, kv_ref, x.cache_off,
                                x.cache_len, x.cache_cap)
    for b in (0, 3):
        for k in ("am", "acc_len", "acc_nodes", "out_tok", "bonus"):
            assert np.array_equal(got[k][b], ref[k][b]), (k, b)
        assert got["status"][b] == 0
    assert np.array_equal(bf16_tensor_bits(kv), kv_ref)  # requests 1 and 2 copied nothing


# ---------------------------------------------------------------------------
# the sweep's largest batch x budget corner: B 64, N 256, K 16, V 163840
# ---------------------------------------------------------------------------


@pytest.fixture(scope="module")
def corner():
    s = synth.kimi_sweep(64, 256, 512)
    x = synth.make_step(s)
    return s, x, oracle.build_tree(x.logp, x.tok, x.root_tok, x.cache_len, s.N)


def test_build_sweep_corner(corner):
    s, x, ref = corner
    assert s.K == 16 and int(ref["n_nodes"].min()) == 256
    _compare_tree(_run_build(x, s.N), ref)


def test_accept_sweep_corner(corner):
    """64 requests x 256 rows x 163840 bf16 logits (5.4 GB), drawn on the GPU
    with a seeded generator (the same bytes go to the oracle, one request at a
    time). Each request gets a planted path to a random node, plus +5 on a
    random child of 70 % of the nodes."""
    s, x, tree = corner
    B, N, V = s.B, s.N, s.V
    g = torch.Generator(device=DEV)
    g.manual_seed(4242)
    logits = torch.randn(B, N, V, generator=g, device=DEV).to(torch.bfloat16)
    rng = np.random.default_rng(99)
    for b in range(B):
        n = int(tree["n_nodes"][b])
        for i in range(n):
            kids = np.flatnonzero(tree["parent"][b, :n] == i)
            if len(kids) and rng.random() < 0.7:
                c = int(kids[rng.integers(len(kids))])
                logits[b, i, int(tree["node_tok"][b, c])] += 5.0
        node = int(rng.integers(1, n))
        path = []
        while node > 0:
            path.append(node)
            node = int(tree["parent"][b, node])
        prev = 0
        for node in path[::-1]:
            logits[b, prev, int(tree["node_tok"][b, node])] = 30.0
            prev = node
    d = step_to_device(x, DEV)
    kv = t_from(x.kv, DEV, True)
    cl = d["cache_len"].clone()
    out = lib.accept_compact(logits, t_from(tree["node_tok"], DEV), t_from(tree["parent"], DEV),
                             t_from(tree["n_nodes"], DEV), kv, d["cache_off"], cl, d["cache_cap"])
    torch.cuda.synchronize()
    got = {k: v.cpu().numpy() for k, v in out.items()}
    kv_got = bf16_tensor_bits(kv)
    kv_ref = x.kv.copy()
    for b in range(B):
        lg = logits[b:b + 1].view(torch.int16).cpu().numpy().view(np.uint16)
        sl = {k: tree[k][b:b + 1] for k in ("node_tok", "parent", "n_nodes")}
        ref = oracle.accept_compact(lg, "bf16", sl["node_tok"], sl["parent"], sl["n_nodes"], kv_ref,
                                    x.cache_off[b:b + 1], x.cache_len[b:b + 1], x.cache_cap[b:b + 1])
        for k in ("am", "acc_len", "acc_nodes", "out_tok", "bonus", "status"):
            assert np.array_equal(got[k][b:b + 1], ref[k]), (k, b)
        assert cl[b].item() == ref["cache_len"][0]
    assert got["acc_len"].min() >= 1
    assert np.array_equal(kv_got, kv_ref)


def test_accept_status_word_timeout_skips_everything():
    """A workspace whose status word holds a timeout (as an argmax kernel that
    gave up a wait on its copies leaves it) makes the call accept nothing:
    every request reports DDT_ERR_TIMEOUT, keeps its cache and cache_len, and
    the row keys are left at zero; after the caller zeroes the workspace the
    same call matches the oracle."""
    s = synth.custom(B=3, D=3, K=3, N=12, H=1, d_l=32, d_r=8, V=4096, L=(3, 7, 11), dtype="bf16", seed=12,
                     accept_p=1.0)
    x, tree, logits = _accept_case(s)
    d = step_to_device(x, DEV)
    kv = t_from(x.kv, DEV, True)
    ws = torch.zeros(lib.accept_compact_workspace_size(s.B, s.N, s.V), dtype=torch.uint8, device=DEV)
    ws[:4].view(torch.int32)[0] = lib.DDT_ERR_TIMEOUT
    cl = d["cache_len"].clone()
    args = (t_from(logits, DEV, True), t_from(tree["node_tok"], DEV), t_from(tree["parent"], DEV),
            t_from(tree["n_nodes"], DEV), kv, d["cache_off"])
    out = lib.accept_compact(*args, cl, d["cache_cap"], workspace=ws)
    torch.cuda.synchronize()
    assert np.all(out["status"].cpu().numpy() == lib.DDT_ERR_TIMEOUT)
    assert np.all(out["acc_len"].cpu().numpy() == 0) and np.array_equal(cl.cpu().numpy(), x.cache_len)
    assert np.array_equal(bf16_tensor_bits(kv), x.kv)
    assert int(ws[256:].view(torch.int64).abs().sum().item()) == 0
    ws.zero_()
    _run_accept_and_compare(s, x, tree, logits)


@pytest.mark.parametrize("B,N,V,pad", [(1, 64, 163840, 0), (4, 128, 163840, 0), (3, 40, 20000, 9)])
def test_accept_leaves_workspace_zero(B, N, V, pad):
    """The argmax hands out its slices through counters in the workspace
    header and reduces every row, pad rows included; after the call the whole
    workspace (status word, counters, every row's key) is zero again, so the
    next call on it starts clean. Two calls in a row give the same outputs.
    (64 and 512 rows take the bulk-copy and the register-fed argmax.)"""
    g = torch.Generator(device=DEV)
    g.manual_seed(B * 1000 + N)
    lg = torch.randn(B, N, V, generator=g, device=DEV).to(torch.bfloat16)
    nt = torch.zeros(B, N, dtype=torch.int32, device=DEV)
    par = torch.full((B, N), -1, dtype=torch.int32, device=DEV)
    par[:, 1:] = 0
    nn = torch.full((B,), N - pad, dtype=torch.int32, device=DEV)
    kv = torch.zeros(B * (N + 8), 64, dtype=torch.bfloat16, device=DEV)
    off = (torch.arange(B, device=DEV) * (N + 8)).to(torch.int64)
    cap = torch.full((B,), N + 8, dtype=torch.int32, device=DEV)
    ws = torch.zeros(lib.accept_compact_workspace_size(B, N, V), dtype=torch.uint8, device=DEV)
    outs = []
    for _ in range(2):
        cl = torch.zeros(B, dtype=torch.int32, device=DEV)
        out = lib.accept_compact(lg, nt, par, nn, kv, off, cl, cap, workspace=ws)
        torch.cuda.synchronize()
        assert int(ws.to(torch.int64).abs().sum().item()) == 0
        outs.append({k: v.cpu().numpy() for k, v in out.items()})
    for k in ("am", "acc_len", "acc_nodes", "out_tok", "bonus", "status"):
        assert np.array_equal(outs[0][k], outs[1][k]), k
    # the argmax itself: every real row against the oracle's (lowest index on ties)
    ref = oracle.row_argmax(lg.float().cpu().numpy())
    am = outs[0]["am"]
    for b in range(B):
        n = N - pad
        assert np.array_equal(am[b, :n], ref[b, :n])
        assert np.all(am[b, n:] == -1)
