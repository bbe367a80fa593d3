"""Helpers shared by the tests: host arrays -> device tensors, guard-banded
output buffers, the tolerance checks the parity bar uses, and the drafters of
the speculative-loop tests."""
import numpy as np
import torch

from ddtree_speculative_decode_b200 import synth

# Float tolerance of the tree-verify attention: max-abs 2e-3 for float32
# outputs; for bf16 outputs max |gpu - oracle| <= 2e-2 * max |oracle| over the
# request's output tensor ("relative to scale", read per request).
TOL_F32_ABS = 2e-3
TOL_BF16_REL = 2e-2
TOL_LSE_ABS = 2e-3


def t_from(arr: np.ndarray, dev, bf16: bool = False) -> torch.Tensor:
    a = np.ascontiguousarray(arr)
    if bf16:
        return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
    return torch.from_numpy(a).to(dev)


def bf16_tensor_bits(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def step_to_device(x: synth.StepInputs, dev) -> dict:
    bf = x.shape.dtype == "bf16"
    return {
        "logp": t_from(x.logp, dev), "tok": t_from(x.tok, dev), "root_tok": t_from(x.root_tok, dev),
        "cache_len": t_from(x.cache_len, dev), "cache_off": t_from(x.cache_off, dev),
        "cache_cap": t_from(x.cache_cap, dev), "kv": t_from(x.kv, dev, bf), "q": t_from(x.q, dev, bf),
    }


def guarded(shape, dtype, dev, fill, guard=64):
    """A tensor of `shape` that is the prefix of a larger buffer whose tail is a
    canary; check_guard(buf) verifies nothing wrote past the end."""
    n = int(np.prod(shape))
    buf = torch.full((n + guard,), fill, dtype=dtype, device=dev)
    return buf[:n].view(*shape), buf


def check_guard(buf: torch.Tensor, n: int, fill):
    tail = buf[n:].cpu()
    assert torch.all(tail == fill), "write past the end of an output buffer"


def widen_out(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def assert_attn_close(got: np.ndarray, ref: np.ndarray, out_bf16: bool, what=""):
    """got / ref: [B, N, H, d_l] (padded rows included)."""
    for b in range(ref.shape[0]):
        err = np.abs(got[b] - ref[b]).max() if ref[b].size else 0.0
        if out_bf16:
            scale = np.abs(ref[b]).max()
            assert err <= TOL_BF16_REL * max(scale, 1e-30), f"{what} request {b}: max err {err} vs scale {scale}"
        else:
            assert err <= TOL_F32_ABS, f"{what} request {b}: max abs err {err}"


def golden_drafter(golden, V, p_hit=1.0, seed=0):
    """Per-depth top-K proposals from a golden continuation (for the
    speculative-loop tests): rank 0 is the golden token with probability
    p_hit; otherwise the golden token sits at a lower rank or is missing.
    Distractors are other in-vocabulary tokens; log-probs are strictly
    decreasing and <= 0. Returns draft(committed, D, K) -> (logp, tok)."""
    rng = np.random.default_rng(seed)

    def draft(committed, D, K):
        lp = np.zeros((D, K), np.float32)
        tk = np.zeros((D, K), np.int32)
        for d in range(D):
            g = int(golden[len(committed) + d])
            others = [t for t in rng.permutation(V)[:K + 1] if t != g][:K]
            r = rng.random()
            if r < p_hit:
                row = [g] + others[:K - 1]
            elif r < p_hit + (1 - p_hit) / 2 and K > 1:
                pos = int(rng.integers(1, K))
                row = others[:pos] + [g] + others[pos:K - 1]
            else:
                row = others[:K]
            tk[d] = row
            lp[d] = -np.arange(K, dtype=np.float32) * 0.75 - (0.0 if r < p_hit else 0.5)
        return lp, tk

    return draft
