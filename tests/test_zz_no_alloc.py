"""The allocation-free accept entry point gives exactly what the workspace
entry point gives.

ddt_accept_compact_noalloc serves callers that cannot allocate device memory
where they verify a tree (they are handed fixed buffers, or must not risk the
device-wide synchronisation cudaMalloc can cause); its scratch is a fixed
array inside the library. This file runs last (pytest collects it after the
other parity tests), so a failure here never hides their results. Two calls in a
row check that the shared array's leftovers from the previous call do not
leak into the next one."""
import numpy as np
import pytest
import torch

import oracle
from ddtree_speculative_decode_b200 import lib, synth
from ddt_testutil import bf16_tensor_bits, step_to_device, t_from

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _case(s):
    x = synth.make_step(s)
    tree = oracle.build_tree(x.logp, x.tok, x.root_tok, x.cache_len, s.N)
    logits = synth.target_logits(s, tree["parent"], tree["node_tok"], tree["n_nodes"])
    return x, tree, logits


def _run(fn, s, x, tree, logits, **kw):
    bf = s.dtype == "bf16"
    d = step_to_device(x, DEV)
    kv = t_from(x.kv, DEV, bf)
    cl = d["cache_len"].clone()
    out = fn(t_from(logits, DEV, bf), t_from(tree["node_tok"], DEV), t_from(tree["parent"], DEV),
             t_from(tree["n_nodes"], DEV), kv, d["cache_off"], cl, d["cache_cap"], **kw)
    torch.cuda.synchronize()
    res = {k: v.cpu().numpy() for k, v in out.items()}
    res["cache_len"] = cl.cpu().numpy()
    res["kv"] = bf16_tensor_bits(kv) if bf else kv.cpu().numpy()
    return res


@pytest.mark.parametrize("name", ["tiny-f32", "kimi-16req"])
def test_noalloc_matches_workspace_entry_point(name):
    s = synth.NAMED[name]()
    x, tree, logits = _case(s)
    ref = _run(lib.accept_compact, s, x, tree, logits)
    for _ in range(2):  # two calls in a row on the shared scratch
        got = _run(lib.accept_compact_noalloc, s, x, tree, logits)
        for k in ("am", "acc_len", "acc_nodes", "out_tok", "bonus", "status", "cache_len"):
            assert np.array_equal(got[k], ref[k]), k
        assert np.array_equal(got["kv"], ref["kv"])
