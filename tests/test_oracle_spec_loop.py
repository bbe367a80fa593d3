"""Pins of the speculative loop on a tiny MLA decoder with random weights: the
DDTree loop (drafter -> build_tree -> one target forward over the tree rows,
attention through verify_attn with the tree's visibility mask on every layer
-> accept walk -> compaction of all layers) reproduces the autoregressive
greedy output token for token, with the step counts the pages print for the
oracle drafter, and leaves the same latent caches behind."""
import os

import numpy as np
import pytest

from oracle import spec_loop
from ddtree_speculative_decode_b200 import synth
from ddt_testutil import golden_drafter as _drafter

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "capstone_ddtree_stats.txt")
PROMPT = [3, 14, 15, 92, 65]


def _golden():
    vals = {}
    for line in open(GOLDEN):
        line = line.strip()
        if line and not line.startswith("#"):
            k, v = line.split()
            vals[k] = v
    return vals


@pytest.fixture(scope="module")
def model():
    return synth.tiny_mla_weights()


def test_oracle_drafter_reproduces_the_pages_statistics(model):
    g = _golden()
    T, blk = int(g["tokens"]), int(g["block_size"])
    ar, _ = spec_loop.ar_generate(model, PROMPT, T + blk)
    dd, steps, _ = spec_loop.ddtree_generate(model, PROMPT, T, _drafter(ar, model["V"]), blk, K=3)
    assert dd[:T] == ar[:T]
    assert steps == int(g["steps"]) == int(g["target_forwards_ddtree"])
    assert len(dd) == int(g["committed"])
    assert "%.2f" % ((len(dd) - 1) / steps) == g["avg_accept"]


def test_compacted_caches_equal_the_autoregressive_ones(model):
    T, blk = 24, 8
    ar, ar_cache = spec_loop.ar_generate(model, PROMPT, T + blk)
    dd, _, dd_cache = spec_loop.ddtree_generate(model, PROMPT, T, _drafter(ar, model["V"]), blk, K=3)
    rows = dd_cache.length
    assert rows == len(PROMPT) + len(dd) - 1  # every committed token but the last root
    assert ar_cache.length >= rows
    for layer in range(dd_cache.n_layers):
        np.testing.assert_allclose(dd_cache.layer(layer)[:rows], ar_cache.layer(layer)[:rows], rtol=1e-9,
                                   atol=1e-12)


@pytest.mark.parametrize("seed", range(5))
def test_noisy_drafters_stay_greedy_exact(model, seed):
    """Branching trees (the golden token at a lower rank, or missing): every
    accepted node must still be the AR token, and rejected branches must leave
    no trace in the cache."""
    T, blk, K = 30, 8, 3
    ar, ar_cache = spec_loop.ar_generate(model, PROMPT, T + blk)
    dd, steps, dd_cache = spec_loop.ddtree_generate(model, PROMPT, T, _drafter(ar, model["V"], 0.6, seed), blk, K)
    assert dd[:T] == ar[:T]
    assert steps < T - 1  # some drafts were accepted
    rows = dd_cache.length
    for layer in range(dd_cache.n_layers):
        np.testing.assert_allclose(dd_cache.layer(layer)[:rows], ar_cache.layer(layer)[:rows], rtol=1e-9,
                                   atol=1e-12)


def test_a_drafter_that_is_always_wrong_commits_one_token_per_step(model):
    T, blk, K = 12, 8, 3
    ar, _ = spec_loop.ar_generate(model, PROMPT, T + blk)
    dd, steps, _ = spec_loop.ddtree_generate(model, PROMPT, T, _drafter(ar, model["V"], p_hit=0.0, seed=3), blk,
                                             K=1)
    assert dd[:T] == ar[:T]
    assert steps == T - 1  # one bonus token per verify step after the prefill's first


@pytest.mark.parametrize("blk,K", [(2, 1), (4, 2), (16, 4)])
def test_other_block_sizes(model, blk, K):
    T = 20
    ar, _ = spec_loop.ar_generate(model, PROMPT, T + blk)
    dd, steps, _ = spec_loop.ddtree_generate(model, PROMPT, T, _drafter(ar, model["V"], 0.8, blk), blk, K)
    assert dd[:T] == ar[:T]


def test_the_gpu_engine_has_no_cpu_path(model):
    import torch

    from ddtree_speculative_decode_b200 import spec_engine
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    with pytest.raises(RuntimeError):
        spec_engine.TinyMLAEngine(model, capacity=64)
