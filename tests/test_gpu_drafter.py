"""GPU parity of ddt_drafter_topk against oracle.drafter_topk: token ids bit
exact (top-k order, ties to the lower index), log-probs within a float32
tolerance, on Kimi-sized rows, odd vocabulary sizes (scalar path), every K
range of the kernel, rows split over several CTAs (a cluster of up to 8 per
row, slices of at least 16384 logits) and heavily tied rows."""
import numpy as np
import pytest
import torch

import oracle
from ddtree_speculative_decode_b200 import lib, synth

pytestmark = pytest.mark.gpu
DEV = "cuda:0"

# float32 log-sum-exp over up to 163840 terms against the oracle's float64 one,
# then one float32 subtraction: a few ulp of |logp| plus the sum's rounding
TOL_ABS, TOL_REL = 2e-5, 2e-6


def _logits(R, V, dtype, seed, sigma=3.0, quant=None):
    rng = np.random.default_rng(seed)
    z = (rng.standard_normal((R, V)) * sigma).astype(np.float32)
    if quant:
        z = (np.round(z / quant) * quant).astype(np.float32)
    if dtype == "bf16":
        bits = synth.f32_to_bf16_bits(z)
        return torch.from_numpy(bits.view(np.int16)).to(DEV).view(torch.bfloat16), synth.bf16_bits_to_f32(bits)
    return torch.from_numpy(z).to(DEV), z


def _check(out, z, K):
    ref_lp, ref_tok, ref_st = oracle.drafter_topk(z.astype(np.float64), K)
    tok = out["tok"].cpu().numpy().reshape(ref_tok.shape)
    lp = out["logp"].cpu().numpy().reshape(ref_lp.shape).astype(np.float64)
    st = out["status"].cpu().numpy().reshape(ref_st.shape)
    assert np.array_equal(st, ref_st)
    assert np.array_equal(tok, ref_tok)
    fin = np.isfinite(ref_lp)
    assert np.array_equal(fin, np.isfinite(lp))
    d = np.abs(lp[fin] - ref_lp[fin])
    assert np.all(d <= TOL_ABS + TOL_REL * np.abs(ref_lp[fin])), d.max()


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("K", [1, 8, 16, 32])
def test_kimi_rows(dtype, K):
    t, z = _logits(8, 163840, dtype, seed=K)
    out = lib.drafter_topk(t, K)
    torch.cuda.synchronize()
    _check(out, z, K)


@pytest.mark.parametrize(
    "V,K",
    [(1, 1), (5, 5), (7, 3), (256, 8), (1001, 16), (4099, 32), (16384, 4), (16392, 5), (40000, 16),
     (65537, 9), (114696, 32), (200000, 8)],
)
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_sizes(V, K, dtype):
    t, z = _logits(5, V, dtype, seed=V + K)
    out = lib.drafter_topk(t, K)
    torch.cuda.synchronize()
    _check(out, z, K)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_ties_go_to_the_lower_index(dtype):
    t, z = _logits(6, 20000, dtype, seed=9, sigma=1.0, quant=0.5)  # thousands of equal values
    out = lib.drafter_topk(t, 32)
    torch.cuda.synchronize()
    _check(out, z, 32)


@pytest.mark.parametrize("V", [40000, 163840, 50001])
def test_ties_and_winners_across_slices(V):
    """Equal maxima in different CTAs' slices go to the lower index; the K
    best all in the last slice, or straddling a slice start."""
    z = np.random.default_rng(V).standard_normal((4, V)).astype(np.float32)
    z[0, [V - 1, V // 2, 3, V // 3 + 1]] = 9.0      # four-way tie across slices
    z[1, V - 20:] = np.linspace(5.0, 8.0, 20, dtype=np.float32)  # all winners last
    C = min(8, (V + 16383) // 16384)
    chunk = ((V + C - 1) // C + 7) // 8 * 8
    for c in range(1, C):                           # around each slice start
        z[2, c * chunk - 2: c * chunk + 2] = 7.0 + c * 0.01
    z[3, :] = 0.0                                   # all equal: ids 0..K-1
    out = lib.drafter_topk(torch.from_numpy(z).to(DEV), 16)
    torch.cuda.synchronize()
    _check(out, z, 16)
    assert list(out["tok"].cpu().numpy()[3]) == list(range(16))


def test_non_finite_in_a_later_slice():
    z = np.random.default_rng(5).standard_normal((3, 100000)).astype(np.float32)
    z[0, 99999] = np.nan
    z[2, 60000] = np.inf
    out = lib.drafter_topk(torch.from_numpy(z).to(DEV), 8)
    torch.cuda.synchronize()
    _check(out, z, 8)
    assert list(out["status"].cpu().numpy()) == [lib.DDT_ERR_INPUT, lib.DDT_OK, lib.DDT_ERR_INPUT]


def test_non_finite_rows():
    z = np.random.default_rng(2).standard_normal((4, 3000)).astype(np.float32)
    z[1, 17] = np.nan
    z[3, 2999] = -np.inf
    out = lib.drafter_topk(torch.from_numpy(z).to(DEV), 8)
    torch.cuda.synchronize()
    _check(out, z, 8)
    st = out["status"].cpu().numpy()
    assert list(st) == [lib.DDT_OK, lib.DDT_ERR_INPUT, lib.DDT_OK, lib.DDT_ERR_INPUT]


def test_feeds_the_tree_build():
    """[B, D, V] logits -> [B, D, K] proposals the build accepts as they are."""
    t, z = _logits(2 * 6, 5000, "bf16", seed=21)
    out = lib.drafter_topk(t.view(2, 6, 5000), 6)
    root = torch.tensor([3, 4], dtype=torch.int32, device=DEV)
    cl = torch.tensor([100, 0], dtype=torch.int32, device=DEV)
    tree = lib.build_tree(out["logp"], out["tok"], root, cl, 32)
    torch.cuda.synchronize()
    assert list(tree["status"].cpu().numpy()) == [lib.DDT_OK, lib.DDT_OK]
    assert list(tree["n_nodes"].cpu().numpy()) == [32, 32]
