"""The speculative loop through the library on a GPU (ddt_build_tree ->
ddt_verify_attn on every layer of a tiny MLA decoder -> ddt_accept_compact
over all layers), against the oracle's loop on the CPU: the same greedy
tokens, DDTree equal to AR, the pages' oracle-drafter statistics, and the
compacted latent caches equal to the AR ones. The oracle's logits keep a top-2
gap of at least 0.017 along these runs (logits of scale about 3.5), far above
float32 error, so the float32 GPU loop must pick the same tokens. This file
sorts after the other GPU test files."""
import numpy as np
import pytest
import torch

from oracle import spec_loop
from ddtree_speculative_decode_b200 import spec_engine, synth
from ddt_testutil import golden_drafter

pytestmark = pytest.mark.gpu
PROMPT = [3, 14, 15, 92, 65]


@pytest.fixture(scope="module")
def weights():
    return synth.tiny_mla_weights()


@pytest.fixture(scope="module")
def ar_ref(weights):
    toks, _ = spec_loop.ar_generate(weights, PROMPT, 40)
    return toks


def test_ar_matches_the_oracle(weights, ar_ref):
    eng = spec_engine.TinyMLAEngine(weights, capacity=128)
    assert eng.ar_generate(PROMPT, 40) == ar_ref


def test_oracle_drafter_statistics(weights, ar_ref):
    eng = spec_engine.TinyMLAEngine(weights, capacity=128)
    dd, steps = eng.ddtree_generate(PROMPT, 24, golden_drafter(ar_ref, weights["V"]), block=8, K=3)
    assert dd[:24] == ar_ref[:24]
    assert steps == 3 and len(dd) == 25


@pytest.mark.parametrize("seed", range(3))
def test_noisy_drafters_stay_greedy_exact(weights, ar_ref, seed):
    eng = spec_engine.TinyMLAEngine(weights, capacity=128)
    dd, steps = eng.ddtree_generate(PROMPT, 30, golden_drafter(ar_ref, weights["V"], 0.6, seed), block=8, K=3)
    assert dd[:30] == ar_ref[:30]
    assert steps < 29
    ar_eng = spec_engine.TinyMLAEngine(weights, capacity=128)
    ar_eng.ar_generate(PROMPT, 33)
    rows = eng.length
    for li in range(eng.n_layers):
        got = eng.layer(li)[:rows].cpu().numpy()
        ref = ar_eng.layer(li)[:rows].cpu().numpy()
        np.testing.assert_allclose(got, ref, rtol=1e-4, atol=1e-5)
    torch.cuda.synchronize()
