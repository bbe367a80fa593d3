"""The speculative decoding loop through the library on a GPU, on a tiny MLA
decoder: every attention call is ddt_verify_attn on the layer's latent pool
(one new row per token in the autoregressive loop; the whole draft tree with
its visibility mask in the DDTree loop), ddt_build_tree turns the drafter's
per-depth proposals into the tree, and ddt_accept_compact walks the target's
greedy choices and compacts every layer's pool.

Sources: capstone page, "The Oracle Drafter" and "The Results: A Perfect
Validation" (with a drafter that proposes the golden continuation, DDTree
reproduces the autoregressive greedy output and commits a whole block per
verify step); AR page, "The Broader Context" (KV cache with post-verify
compaction); "the_validation_pivot", "Assumptions Embedded in This Message"
(the tiny model's sizes).

The model around the library is torch arithmetic on the GPU: a pre-norm
decoder with RMS normalisation without weights, absorbed MLA attention (the
query's no-rope part folded through the key up-projection, the latent output
through the value up-projection), interleaved rotary embedding with base
10000 on the rope parts, a ReLU MLP and an LM head. There is no CPU path.
"""
from __future__ import annotations

import numpy as np
import torch

from . import lib


def _rms(x):
    return x * torch.rsqrt((x * x).mean(-1, keepdim=True) + 1e-6)


def _rope(x, pos, base=10000.0):
    """Rotate consecutive pairs of the last axis by pos * base^(-2k / d)."""
    d = x.shape[-1]
    inv = base ** (-torch.arange(0, d, 2, dtype=torch.float64, device=x.device) / d)
    ang = pos.to(torch.float64).reshape((-1,) + (1,) * (x.dim() - 1)) * inv
    c, s = torch.cos(ang).to(x.dtype), torch.sin(ang).to(x.dtype)
    xe, xo = x[..., 0::2], x[..., 1::2]
    out = torch.empty_like(x)
    out[..., 0::2] = xe * c - xo * s
    out[..., 1::2] = xe * s + xo * c
    return out


class TinyMLAEngine:
    """One request's decoder state: weights on the device and one latent pool
    per layer (capacity rows each, stacked at a layer stride), float32."""

    def __init__(self, weights: dict, capacity: int, device: str = "cuda:0"):
        if not torch.cuda.is_available():
            raise RuntimeError("TinyMLAEngine needs a CUDA device (the library has no CPU path)")
        lib.load()
        self.dev = torch.device(device)

        def f(a):
            return torch.as_tensor(np.asarray(a, np.float32), device=self.dev)

        self.embed, self.w_vocab = f(weights["embed"]), f(weights["w_vocab"])
        self.layers = [{k: f(v) for k, v in lw.items()} for lw in weights["layers"]]
        self.V, self.H = int(weights["V"]), int(weights["H"])
        self.d_l, self.d_r, self.d_v = int(weights["d_latent"]), int(weights["d_rope"]), int(weights["d_v"])
        self.scale = float(weights["scale"])
        self.n_layers, self.stride = len(self.layers), int(capacity)
        self.kv = torch.zeros(self.n_layers * self.stride, self.d_l + self.d_r, dtype=torch.float32,
                              device=self.dev)
        self.length = 0  # committed rows in every layer's pool
        self.off = torch.zeros(1, dtype=torch.int64, device=self.dev)
        self.cap = torch.tensor([self.stride], dtype=torch.int32, device=self.dev)

    def layer(self, li: int) -> torch.Tensor:
        return self.kv[li * self.stride:(li + 1) * self.stride]

    def _i32(self, v):
        return torch.tensor([int(v)], dtype=torch.int32, device=self.dev)

    def forward_rows(self, toks, pos, mask, n):
        """Target forward of n rows after the committed ones: row t writes its
        latent row at pool row length + t on every layer and attends to the
        committed rows plus the rows its mask selects. toks [n] int64, pos [n],
        mask [1, n, ceil(n / 32)] int32. Returns float32 logits [n, V]."""
        L = self.length
        if not (1 <= n and L + n <= self.stride):
            raise ValueError(f"rows [{L}, {L + n}) do not fit the pool of {self.stride} rows")
        dl, H = self.d_l, self.H
        cl, nn = self._i32(L), self._i32(n)
        x = self.embed[toks]
        for li, lw in enumerate(self.layers):
            h = _rms(x)
            pool = self.layer(li)
            pool[L:L + n, :dl] = h @ lw["w_dkv"].T
            pool[L:L + n, dl:] = _rope(h @ lw["w_kr"].T, pos)
            qn = torch.einsum("hkd,nd->nhk", lw["w_q"], h)
            qr = _rope(torch.einsum("hkd,nd->nhk", lw["w_qr"], h), pos)
            q = torch.cat([torch.einsum("hkl,nhk->nhl", lw["w_uk"], qn), qr], dim=-1).unsqueeze(0).contiguous()
            out, _ = lib.verify_attn(q, pool, self.off, cl, mask, nn, dl, self.d_r, self.scale, L, want_lse=False)
            o = torch.einsum("hvl,nhl->nhv", lw["w_uv"], out[0]).reshape(n, H * self.d_v)
            x = x + o @ lw["w_o"].T
            x = x + torch.relu(_rms(x) @ lw["w_1"].T) @ lw["w_2"].T
        return _rms(x) @ self.w_vocab.T

    def _one_row(self, tok: int) -> int:
        toks = torch.tensor([int(tok)], dtype=torch.int64, device=self.dev)
        pos = torch.tensor([self.length], dtype=torch.int32, device=self.dev)
        mask = torch.ones((1, 1, 1), dtype=torch.int32, device=self.dev)
        lg = self.forward_rows(toks, pos, mask, 1)
        self.length += 1
        return int(torch.argmax(lg[0]).item())  # the first index among equal maxima

    def prefill(self, prompt) -> int:
        nxt = None
        for t in prompt:
            nxt = self._one_row(t)
        return nxt

    def ar_generate(self, prompt, T: int) -> list:
        """Greedy autoregressive decoding: T tokens, one forward per token."""
        out = [self.prefill(prompt)]
        while len(out) < T:
            out.append(self._one_row(out[-1]))
        return out

    def ddtree_generate(self, prompt, T: int, drafter, block: int, K: int):
        """DDTree greedy decoding: per verify step a draft tree of `block` rows
        from drafter(committed, block - 1, K) -> (logp [D, K], tok [D, K]),
        one forward over the tree rows, the accept walk and the compaction of
        every layer. Returns (committed tokens, verify steps)."""
        committed = [self.prefill(prompt)]
        steps = 0
        while len(committed) < T:
            lp, tk = drafter(committed, block - 1, K)
            if tk.min() < 0 or tk.max() >= self.V:
                raise ValueError("drafter proposed a token outside the vocabulary")
            L = self.length
            if L + block > self.stride:
                raise ValueError("the pool cannot hold another tree")
            tree = lib.build_tree(torch.as_tensor(np.asarray(lp, np.float32)[None], device=self.dev),
                                  torch.as_tensor(np.asarray(tk, np.int32)[None], device=self.dev),
                                  self._i32(committed[-1]), self._i32(L), block)
            n = int(tree["n_nodes"][0].item())
            if int(tree["status"][0].item()) != lib.DDT_OK or not 1 <= n <= block:
                raise RuntimeError("tree build reported an error")
            logits = torch.zeros((1, block, self.V), dtype=torch.float32, device=self.dev)
            logits[0, :n] = self.forward_rows(tree["node_tok"][0, :n].long(), tree["pos"][0, :n],
                                              tree["mask"][:, :n, :(n + 31) // 32].contiguous(), n)
            cl = self._i32(L)
            acc = lib.accept_compact(logits, tree["node_tok"], tree["parent"], tree["n_nodes"], self.kv, self.off,
                                     cl, self.cap, n_layers=self.n_layers, layer_stride_rows=self.stride)
            if int(acc["status"][0].item()) != lib.DDT_OK:
                raise RuntimeError("accept reported an error")
            a = int(acc["acc_len"][0].item())
            committed += [int(t) for t in acc["out_tok"][0, :a + 1].cpu().tolist()]
            self.length = int(cl[0].item())
            steps += 1
        return committed, steps
