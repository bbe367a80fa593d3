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
