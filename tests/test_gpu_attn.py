"""GPU parity of ddt_verify_attn against the oracle: every row on the tiny
float32 workload and on small edge cases (empty / short caches, budgets around
the 32-bit mask word, pad rows), sampled rows at the Kimi-shaped sizes, with
the float tolerance the parity bar states (tests/ddt_testutil.py)."""
import numpy as np
import pytest
import torch

import oracle
from ddtree_speculative_decode_b200 import lib, synth
from ddt_testutil import (TOL_LSE_ABS, assert_attn_close, step_to_device, t_from, widen_out)

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _attn(s: synth.Shape, x: synth.StepInputs, tree: dict, out_dtype=None, rows=None):
    d = step_to_device(x, DEV)
    mask = t_from(tree["mask"].view(np.int32), DEV)
    nn = t_from(tree["n_nodes"], DEV)
    out, lse = lib.verify_attn(d["q"], d["kv"], d["cache_off"], d["cache_len"], mask, nn, s.d_l, s.d_r, s.scale,
                               int(max(s.L)), out_dtype=out_dtype)
    torch.cuda.synchronize()
    ref, ref_lse = oracle.verify_attn(x.q, x.kv, x.cache_off, x.cache_len, tree["mask"], tree["n_nodes"], s.H, s.d_l,
                                      s.d_r, s.scale, s.dtype, rows=rows)
    return widen_out(out), lse.cpu().numpy().astype(np.float64), ref, ref_lse


def _check(got, glse, ref, rlse, bf16_out, rows=None):
    if rows is not None:
        sel = np.zeros(ref.shape[:2], bool)
        for b, i in rows:
            sel[b, i] = True
        got = np.where(sel[:, :, None, None], got, 0.0)
        ref = np.where(sel[:, :, None, None], ref, 0.0)
        glse = np.where(sel[:, :, None], glse, -np.inf)
        rlse = np.where(sel[:, :, None], rlse, -np.inf)
    assert_attn_close(got, ref, bf16_out)
    fin = np.isfinite(rlse)
    assert np.array_equal(fin, np.isfinite(glse)), "pad-row lse"
    if fin.any():
        assert np.abs(glse[fin] - rlse[fin]).max() <= TOL_LSE_ABS


def _tree(x, s):
    return oracle.build_tree(x.logp, x.tok, x.root_tok, x.cache_len, s.N)


def test_attn_tiny_f32():
    s = synth.tiny_f32()
    x = synth.make_step(s)
    g, gl, r, rl = _attn(s, x, _tree(x, s))
    _check(g, gl, r, rl, False)


@pytest.mark.parametrize("L", [0, 1, 63, 64, 65, 200])
@pytest.mark.parametrize("N", [1, 2, 31, 33])
def test_attn_f32_edges(L, N):
    s = synth.custom(B=2, D=4, K=3, N=N, H=3, d_l=64, d_r=16, V=64, L=(L, max(0, L - 1)), seed=L * 100 + N)
    x = synth.make_step(s)
    t = _tree(x, s)
    g, gl, r, rl = _attn(s, x, t)
    _check(g, gl, r, rl, False)


def test_attn_empty_tree_rows_are_zero():
    s = synth.custom(B=2, D=3, K=2, N=8, H=2, d_l=64, d_r=16, V=64, L=(10, 12), seed=5)
    x = synth.make_step(s)
    t = _tree(x, s)
    t["n_nodes"][1] = 0
    g, gl, r, rl = _attn(s, x, t)
    _check(g, gl, r, rl, False)
    assert np.all(g[1] == 0) and np.all(np.isneginf(gl[1]))


def _sample_rows(s: synth.Shape, tree, per_req, seed):
    rng = np.random.default_rng(seed)
    rows = []
    for b in range(s.B):
        n = int(tree["n_nodes"][b])
        pick = {0, n - 1} | set(int(v) for v in rng.integers(0, n, size=per_req))
        rows += [(b, i) for i in sorted(pick)]
    return rows


@pytest.mark.parametrize("name,per_req,out_dtype", [
    ("kimi-1req", 64, torch.bfloat16),
    ("kimi-1req", 6, torch.float32),
    ("kimi-16req", 3, torch.bfloat16),
    ("kimi-4req-32k", 4, torch.bfloat16),
])
def test_attn_kimi_sampled(name, per_req, out_dtype):
    s = synth.NAMED[name]()
    x = synth.make_step(s)
    t = _tree(x, s)
    rows = _sample_rows(s, t, per_req, 17)
    g, gl, r, rl = _attn(s, x, t, out_dtype=out_dtype, rows=rows)
    _check(g, gl, r, rl, out_dtype == torch.bfloat16, rows=rows)
    # pad rows (beyond n_nodes) are zero on the GPU side
    for b in range(s.B):
        n = int(t["n_nodes"][b])
        assert np.all(g[b, n:] == 0)


@pytest.mark.parametrize("L", [0, 1, 63, 64, 65, 127, 129])
@pytest.mark.parametrize("N", [1, 3, 32, 33])
def test_attn_bf16_small(L, N):
    s = synth.custom(B=2, D=5, K=3, N=N, H=64, d_l=512, d_r=64, V=64, L=(L, L + 70), dtype="bf16",
                     kv_scale=0.1, scale=1.0 / np.sqrt(192.0), seed=7 * L + N)
    x = synth.make_step(s)
    t = _tree(x, s)
    g, gl, r, rl = _attn(s, x, t, out_dtype=torch.bfloat16)
    _check(g, gl, r, rl, True)


@pytest.mark.parametrize("L,maxL", [(300, 20000), (0, 5000), (700, 3000)])
def test_attn_bf16_many_splits(L, maxL):
    """A generous max_cache_len makes the launch split every request's keys
    into many slices, most of them empty: the split partials and the combine
    step must still give the oracle's answer."""
    s = synth.custom(B=2, D=4, K=4, N=24, H=64, d_l=512, d_r=64, V=64, L=(L, L + 33), dtype="bf16",
                     kv_scale=0.1, scale=1.0 / np.sqrt(192.0), seed=L + 1)
    x = synth.make_step(s)
    t = _tree(x, s)
    d = step_to_device(x, DEV)
    mask = t_from(t["mask"].view(np.int32), DEV)
    nn = t_from(t["n_nodes"], DEV)
    ws = torch.zeros(lib.verify_attn_workspace_size(s.B, s.N, s.H, 512, 64, maxL, torch.bfloat16), dtype=torch.uint8,
                     device=DEV)
    assert ws.numel() > 256  # split partials are in use
    out, lse = lib.verify_attn(d["q"], d["kv"], d["cache_off"], d["cache_len"], mask, nn, 512, 64, s.scale, maxL,
                               workspace=ws)
    torch.cuda.synchronize()
    assert lib.verify_attn_status(ws) == 0
    ref, rl = oracle.verify_attn(x.q, x.kv, x.cache_off, x.cache_len, t["mask"], t["n_nodes"], s.H, 512, 64, s.scale,
                                 "bf16")
    _check(widen_out(out), lse.cpu().numpy().astype(np.float64), ref, rl, True)


def test_attn_bf16_status_word_stays_zero():
    s = synth.kimi_1req()
    x = synth.make_step(s)
    t = _tree(x, s)
    d = step_to_device(x, DEV)
    ws = torch.zeros(lib.verify_attn_workspace_size(1, 64, 64, 512, 64, 4096, torch.bfloat16), dtype=torch.uint8,
                     device=DEV)
    for _ in range(3):
        lib.verify_attn(d["q"], d["kv"], d["cache_off"], d["cache_len"], t_from(t["mask"].view(np.int32), DEV),
                        t_from(t["n_nodes"], DEV), 512, 64, s.scale, 4096, workspace=ws)
    torch.cuda.synchronize()
    assert lib.verify_attn_status(ws) == lib.DDT_OK


def test_attn_bf16_two_splits_in_one_cluster():
    """Two key splits put both splits of a row tile in one 4-CTA cluster and
    merge them through distributed shared memory. Request 0 has a single key
    tile (its second split is idle) and pad row tiles (n_nodes cut to 20);
    request 1 uses both splits."""
    s = synth.custom(B=2, D=4, K=4, N=32, H=64, d_l=512, d_r=64, V=64, L=(0, 1500), dtype="bf16", kv_scale=0.1,
                     scale=1.0 / np.sqrt(192.0), seed=11)
    x = synth.make_step(s)
    t = _tree(x, s)
    t["n_nodes"][0] = 20
    maxL = 2000
    d = step_to_device(x, DEV)
    mask = t_from(t["mask"].view(np.int32), DEV)
    nn = t_from(t["n_nodes"], DEV)
    ws = torch.zeros(lib.verify_attn_workspace_size(s.B, s.N, s.H, 512, 64, maxL, torch.bfloat16), dtype=torch.uint8,
                     device=DEV)
    assert ws.numel() > 256  # the launch splits the keys
    for _ in range(2):
        out, lse = lib.verify_attn(d["q"], d["kv"], d["cache_off"], d["cache_len"], mask, nn, 512, 64, s.scale, maxL,
                                   workspace=ws)
    torch.cuda.synchronize()
    assert lib.verify_attn_status(ws) == 0
    ref, rl = oracle.verify_attn(x.q, x.kv, x.cache_off, x.cache_len, t["mask"], t["n_nodes"], s.H, 512, 64, s.scale,
                                 "bf16")
    got = widen_out(out)
    _check(got, lse.cpu().numpy().astype(np.float64), ref, rl, True)
    assert np.all(got[0, 20:] == 0) and np.all(np.isneginf(lse.cpu().numpy()[0, 20:]))


# ---------------------------------------------------------------------------
# budgets past 128 rows (mask words 5..8), the sweep's long contexts and
# large batches
# ---------------------------------------------------------------------------


@pytest.mark.parametrize("N,L", [(129, 300), (200, 70), (256, 0), (256, 1000)])
def test_attn_bf16_wide_masks(N, L):
    """Every row of budgets 129..256 (the tree part of the keys spans five to
    eight 32-bit mask words), with the sweep's drafter shape (depth 8,
    top-16)."""
    s = synth.custom(B=2, D=8, K=16, N=N, H=64, d_l=512, d_r=64, V=64, L=(L, L + 37), dtype="bf16",
                     kv_scale=0.1, scale=1.0 / np.sqrt(192.0), seed=N * 10 + L)
    x = synth.make_step(s)
    t = _tree(x, s)
    assert int(t["n_nodes"].min()) == N
    g, gl, r, rl = _attn(s, x, t, out_dtype=torch.bfloat16)
    _check(g, gl, r, rl, True)


@pytest.mark.parametrize("B,N,L,per_req", [
    (1, 256, 4096, 24),
    (1, 64, 65536, 6),
    (4, 64, 65536, 3),
    (64, 16, 4096, 2),
    (64, 256, 512, 2),
])
def test_attn_sweep_sampled(B, N, L, per_req):
    """Sweep points (Kimi shapes) on sampled rows: the first, the last and
    random nodes of every request, all heads."""
    s = synth.kimi_sweep(B, N, L)
    x = synth.make_step(s)
    t = _tree(x, s)
    rows = _sample_rows(s, t, per_req, 23)
    g, gl, r, rl = _attn(s, x, t, out_dtype=torch.bfloat16, rows=rows)
    _check(g, gl, r, rl, True, rows=rows)


# ---------------------------------------------------------------------------
# device-side guards
# ---------------------------------------------------------------------------


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_attn_pool_bounds(dtype):
    """A request whose rows run past the pool (or whose node count exceeds
    N) reads nothing: DDT_ERR_BOUNDS, every row zero with lse -inf; the other
    requests are unaffected."""
    bf = dtype == "bf16"
    s = synth.custom(B=3, D=4, K=3, N=12, H=64 if bf else 4, d_l=512 if bf else 64, d_r=64 if bf else 16, V=64,
                     L=(40, 77, 300), dtype=dtype, kv_scale=0.1 if bf else 1.0,
                     scale=1.0 / np.sqrt(192.0 if bf else 24.0), seed=31)
    x = synth.make_step(s)
    t = _tree(x, s)
    d = step_to_device(x, DEV)
    off = x.cache_off.copy()
    off[1] = x.kv.shape[0] - 50     # rows [off, off + 77 + 12) run past the pool
    nn = t["n_nodes"].copy()
    nn[2] = s.N + 1
    st = torch.full((3,), -5, dtype=torch.int32, device=DEV)
    out, lse = lib.verify_attn(d["q"], d["kv"], t_from(off, DEV), d["cache_len"], t_from(t["mask"].view(np.int32), DEV),
                               t_from(nn, DEV), s.d_l, s.d_r, s.scale, 300, status=st)
    torch.cuda.synchronize()
    assert st.cpu().tolist() == [lib.DDT_OK, lib.DDT_ERR_BOUNDS, lib.DDT_ERR_BOUNDS]
    keep = t["n_nodes"].copy()
    keep[[1, 2]] = 0  # the oracle's pad rows: zeros, lse -inf
    ref, rl = oracle.verify_attn(x.q, x.kv, x.cache_off, x.cache_len, t["mask"], keep, s.H, s.d_l, s.d_r, s.scale,
                                 dtype)
    _check(widen_out(out), lse.cpu().numpy().astype(np.float64), ref, rl, bf)


def test_attn_bounded_wait_times_out():
    """The bounded waits end with DDT_ERR_TIMEOUT instead of spinning. With the
    limit at 10 ms and the split-merge 'published' counters pre-set to a value
    the splits can never reach, each elected merger gives up its wait: the
    status word reads DDT_ERR_TIMEOUT and its rows are written as zeros. A
    second call on that workspace does no work (pad rows only, at once); after
    the caller zeroes the workspace a call matches the oracle again."""
    s = synth.custom(B=2, D=4, K=4, N=24, H=64, d_l=512, d_r=64, V=64, L=(300, 333), dtype="bf16", kv_scale=0.1,
                     scale=1.0 / np.sqrt(192.0), seed=301)
    maxL = 20000  # many key splits: merged through the workspace counters
    x = synth.make_step(s)
    t = _tree(x, s)
    d = step_to_device(x, DEV)
    mask = t_from(t["mask"].view(np.int32), DEV)
    nn = t_from(t["n_nodes"], DEV)
    ws = torch.zeros(lib.verify_attn_workspace_size(s.B, s.N, s.H, 512, 64, maxL, torch.bfloat16), dtype=torch.uint8,
                     device=DEV)
    rowtiles = (s.N * s.H + 127) // 128
    cnt = ws[256:256 + s.B * rowtiles * 2 * 2 * 4].view(torch.int32).view(-1, 2)
    ref, rl = oracle.verify_attn(x.q, x.kv, x.cache_off, x.cache_len, t["mask"], t["n_nodes"], s.H, 512, 64, s.scale,
                                 "bf16")

    def call():
        o, l = lib.verify_attn(d["q"], d["kv"], d["cache_off"], d["cache_len"], mask, nn, 512, 64, s.scale, maxL,
                               workspace=ws)
        torch.cuda.synchronize()
        return widen_out(o), l.cpu().numpy()

    prev = lib.set_wait_limit_ns(10_000_000)
    try:
        cnt[:, 1] = 1 << 30
        got, gl = call()
        assert lib.verify_attn_status(ws) == lib.DDT_ERR_TIMEOUT
        assert np.all(got == 0) and np.all(np.isneginf(gl))  # every row tile's merger gave up
        got, gl = call()  # the status word still holds the timeout: no work
        assert lib.verify_attn_status(ws) == lib.DDT_ERR_TIMEOUT
        assert np.all(got == 0) and np.all(np.isneginf(gl))
    finally:
        lib.set_wait_limit_ns(prev)
    ws.zero_()
    got, gl = call()
    assert lib.verify_attn_status(ws) == lib.DDT_OK
    _check(got, gl.astype(np.float64), ref, rl, True)
