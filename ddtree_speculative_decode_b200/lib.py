"""ctypes binding of libddt.so (C ABI in include/ddt.h).

Argument marshalling only: tensors are checked for device, dtype, shape and
contiguity, then their device pointers and the current CUDA stream go to the
library. Every step of the tree-verify path runs in the library's kernels;
there is no Python or CPU fallback -- if libddt.so cannot be loaded, every
call raises.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libddt.so")

(DDT_OK, DDT_ERR_INVALID_ARG, DDT_ERR_UNSUPPORTED, DDT_ERR_CAPACITY, DDT_ERR_INPUT, DDT_ERR_CUDA, DDT_ERR_TIMEOUT,
 DDT_ERR_BOUNDS) = range(8)
DDT_F32, DDT_BF16 = 0, 1

EXPORTS = (
    "ddt_status_string",
    "ddt_version",
    "ddt_set_wait_limit_ns",
    "ddt_build_tree",
    "ddt_verify_attn_workspace_size",
    "ddt_verify_attn",
    "ddt_accept_compact_workspace_size",
    "ddt_accept_compact",
    "ddt_accept_compact_noalloc",
    "ddt_accept_compact_lmhead",
    "ddt_drafter_topk",
)

_lib = None


class DDTError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {status_string(status)} ({status})")
        self.status = status


def load(path: Optional[str] = None) -> ctypes.CDLL:
    """Load libddt.so (built in-tree by ddtree_speculative_decode_b200.build)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"libddt.so not found at {p}; build it with "
                           "`python -m ddtree_speculative_decode_b200.build`")
    lib = ctypes.CDLL(p)
    vp, i32, i64, f32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    lib.ddt_status_string.restype = ctypes.c_char_p
    lib.ddt_status_string.argtypes = [i32]
    lib.ddt_version.restype = i32
    lib.ddt_version.argtypes = []
    lib.ddt_set_wait_limit_ns.restype = ctypes.c_uint64
    lib.ddt_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    lib.ddt_build_tree.restype = i32
    lib.ddt_build_tree.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.ddt_verify_attn_workspace_size.restype = sz
    lib.ddt_verify_attn_workspace_size.argtypes = [i32, i32, i32, i32, i32, i32, i32]
    lib.ddt_verify_attn.restype = i32
    lib.ddt_verify_attn.argtypes = [vp, vp, i64, vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, i32, i32, i32,
                                    vp, vp, vp, vp, sz, vp]
    lib.ddt_accept_compact_workspace_size.restype = sz
    lib.ddt_accept_compact_workspace_size.argtypes = [i32, i32, i32]
    lib.ddt_accept_compact.restype = i32
    lib.ddt_accept_compact.argtypes = [vp, i32, i32, vp, vp, vp, i32, i32, vp, i64, i32, i32, i32, i64, vp, vp,
                                       vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.ddt_accept_compact_noalloc.restype = i32
    lib.ddt_accept_compact_noalloc.argtypes = [vp, i32, i32, vp, vp, vp, i32, i32, vp, i64, i32, i32, i32, i64, vp,
                                               vp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.ddt_accept_compact_lmhead.restype = i32
    lib.ddt_accept_compact_lmhead.argtypes = [vp, vp, i32, i32, vp, vp, vp, i32, i32, vp, i64, i32, i32, i32, i64,
                                              vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.ddt_drafter_topk.restype = i32
    lib.ddt_drafter_topk.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp, vp]
    if path is None:
        _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().ddt_status_string(int(status)).decode()


def version() -> int:
    return int(load().ddt_version())


def set_wait_limit_ns(ns: int) -> int:
    """ddt_set_wait_limit_ns: wall-clock limit of the kernels' bounded waits
    for calls issued from now on (0: the 2 s default). Returns the previous
    limit."""
    return int(load().ddt_set_wait_limit_ns(int(ns)))


# ---------------------------------------------------------------------------
# marshalling helpers
# ---------------------------------------------------------------------------


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(t: torch.Tensor, name: str, dtype, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a tensor")
    if not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise TypeError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")


def _device(*tensors, stream=None):
    """A context that makes the one CUDA device every tensor of a call lives
    on (and the explicit stream, if any, belongs to) current for the launch;
    nothing is switched when it is current already (as inside a graph
    capture on that device)."""
    devs = {t.device for t in tensors if t is not None}
    if len(devs) != 1:
        raise ValueError(f"tensors of one call must share a CUDA device, got {sorted(map(str, devs))}")
    dev = devs.pop()
    if stream is not None and stream.device != dev:
        raise ValueError(f"stream on {stream.device}, tensors on {dev}")
    if dev.index is None or dev.index == torch.cuda.current_device():
        return contextlib.nullcontext()
    return torch.cuda.device(dev)


def _check_out(out: dict, spec: dict):
    """Caller-supplied output tensors: name -> (dtype, shape)."""
    for name, (dtype, shape) in spec.items():
        if name not in out:
            raise ValueError(f"out: missing {name}")
        _check(out[name], f"out[{name}]", dtype, shape)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return DDT_F32
    if t.dtype == torch.bfloat16:
        return DDT_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _raise(fn: str, st: int):
    if st != DDT_OK:
        raise DDTError(fn, st)


# ---------------------------------------------------------------------------
# the three calls
# ---------------------------------------------------------------------------


def drafter_topk(logits: torch.Tensor, K: int, out: Optional[dict] = None, stream=None) -> dict:
    """ddt_drafter_topk. logits [..., V] f32 / bf16 (e.g. [B, D, V]); returns
    logp [..., K] f32, tok [..., K] i32 (build_tree's inputs) and status [...]."""
    _check(logits, "logits", (torch.float32, torch.bfloat16))
    lead, V = tuple(logits.shape[:-1]), logits.shape[-1]
    R = 1
    for d in lead:
        R *= d
    dev = logits.device
    if out is None:
        out = {"logp": torch.empty(*lead, K, dtype=torch.float32, device=dev),
               "tok": torch.empty(*lead, K, dtype=torch.int32, device=dev),
               "status": torch.empty(*lead, dtype=torch.int32, device=dev)}
    _check_out(out, {"logp": (torch.float32, lead + (K,)), "tok": (torch.int32, lead + (K,)),
                     "status": (torch.int32, lead)})
    with _device(logits, *out.values(), stream=stream):
        st = load().ddt_drafter_topk(_ptr(logits), _dt(logits), V, R, K, _ptr(out["logp"]), _ptr(out["tok"]),
                                     _ptr(out["status"]), _stream(stream))
    _raise("ddt_drafter_topk", st)
    return out


def build_tree(logp: torch.Tensor, tok: torch.Tensor, root_tok: torch.Tensor, cache_len: torch.Tensor, N: int,
               out: Optional[dict] = None, stream=None) -> dict:
    """ddt_build_tree. logp [B, D, K] f32, tok [B, D, K] i32, root_tok / cache_len
    [B] i32. Returns node_tok, parent, depth, pos [B, N] i32, score [B, N] f32,
    mask [B, N, W] i32 (bit patterns of uint32), n_nodes [B], status [B]."""
    B, D, K = logp.shape
    _check(logp, "logp", torch.float32)
    _check(tok, "tok", torch.int32, (B, D, K))
    _check(root_tok, "root_tok", torch.int32, (B,))
    _check(cache_len, "cache_len", torch.int32, (B,))
    dev = logp.device
    W = (N + 31) // 32
    if out is None:
        out = alloc_tree(B, N, dev)
    i32 = torch.int32
    _check_out(out, {"node_tok": (i32, (B, N)), "parent": (i32, (B, N)), "depth": (i32, (B, N)),
                     "pos": (i32, (B, N)), "score": (torch.float32, (B, N)), "mask": (i32, (B, N, W)),
                     "n_nodes": (i32, (B,)), "status": (i32, (B,))})
    with _device(logp, tok, root_tok, cache_len, *out.values(), stream=stream):
        st = load().ddt_build_tree(_ptr(logp), _ptr(tok), _ptr(root_tok), _ptr(cache_len), B, D, K, N,
                                   _ptr(out["node_tok"]), _ptr(out["parent"]), _ptr(out["depth"]),
                                   _ptr(out["pos"]), _ptr(out["score"]), _ptr(out["mask"]), _ptr(out["n_nodes"]),
                                   _ptr(out["status"]), _stream(stream))
    _raise("ddt_build_tree", st)
    return out


def alloc_tree(B: int, N: int, device) -> dict:
    W = (N + 31) // 32
    i32 = dict(dtype=torch.int32, device=device)
    return {
        "node_tok": torch.empty(B, N, **i32), "parent": torch.empty(B, N, **i32),
        "depth": torch.empty(B, N, **i32), "pos": torch.empty(B, N, **i32),
        "score": torch.empty(B, N, dtype=torch.float32, device=device),
        "mask": torch.empty(B, N, W, **i32), "n_nodes": torch.empty(B, **i32),
        "status": torch.empty(B, **i32),
    }


def verify_attn_status(workspace: torch.Tensor) -> int:
    """Device status word of a verify-attention workspace (DDT_OK or
    DDT_ERR_TIMEOUT); reading it synchronises with the device."""
    return int(workspace[:4].view(torch.int32).item())


def verify_attn_workspace_size(B: int, N: int, H: int, d_l: int, d_r: int, max_cache_len: int,
                               in_dtype: torch.dtype) -> int:
    return int(load().ddt_verify_attn_workspace_size(B, N, H, d_l, d_r, max_cache_len,
                                                     DDT_BF16 if in_dtype == torch.bfloat16 else DDT_F32))


def verify_attn(q: torch.Tensor, kv: torch.Tensor, cache_off: torch.Tensor, cache_len: torch.Tensor,
                mask: torch.Tensor, n_nodes: torch.Tensor, d_l: int, d_r: int, scale: float, max_cache_len: int,
                out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None, want_lse: bool = True,
                out_dtype: Optional[torch.dtype] = None, workspace: Optional[torch.Tensor] = None,
                status: Optional[torch.Tensor] = None, stream=None):
    """ddt_verify_attn. q [B, N, H, d_qk], kv [rows, d_qk] (same dtype, f32 or
    bf16), cache_off [B] i64, cache_len / n_nodes [B] i32, mask [B, N, W] i32.
    status (optional, [B] i32) receives each request's device status (DDT_OK,
    or DDT_ERR_BOUNDS for rows outside the pool).
    Returns (out [B, N, H, d_l], lse [B, N, H] f32 or None)."""
    B, N, H, d_qk = q.shape
    assert d_qk == d_l + d_r
    _check(q, "q", (torch.float32, torch.bfloat16))
    _check(kv, "kv", q.dtype)
    if kv.dim() != 2 or kv.shape[1] != d_qk:
        raise ValueError("kv: expected [rows, d_qk]")
    _check(cache_off, "cache_off", torch.int64, (B,))
    _check(cache_len, "cache_len", torch.int32, (B,))
    _check(mask, "mask", torch.int32, (B, N, (N + 31) // 32))
    _check(n_nodes, "n_nodes", torch.int32, (B,))
    odt = out_dtype or q.dtype
    if out is None:
        out = torch.empty(B, N, H, d_l, dtype=odt, device=q.device)
    _check(out, "out", odt, (B, N, H, d_l))
    if lse is None and want_lse:
        lse = torch.empty(B, N, H, dtype=torch.float32, device=q.device)
    if lse is not None:
        _check(lse, "lse", torch.float32, (B, N, H))
    if status is not None:
        _check(status, "status", torch.int32, (B,))
    need = verify_attn_workspace_size(B, N, H, d_l, d_r, max_cache_len, q.dtype)
    if workspace is None and need > 0:
        workspace = torch.zeros(need, dtype=torch.uint8, device=q.device)  # status word must start at 0
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with _device(q, kv, cache_off, cache_len, mask, n_nodes, out, lse, status, workspace, stream=stream):
        st = load().ddt_verify_attn(_ptr(q), _ptr(kv), kv.shape[0], _ptr(cache_off), _ptr(cache_len), _ptr(mask),
                                    _ptr(n_nodes), B, N, H, d_l, d_r, float(scale), int(max_cache_len), _dt(q),
                                    _dt(out), _ptr(out), _ptr(lse), _ptr(status), _ptr(workspace), wbytes,
                                    _stream(stream))
    _raise("ddt_verify_attn", st)
    return out, lse


def accept_compact_workspace_size(B: int, N: int, V: int) -> int:
    return int(load().ddt_accept_compact_workspace_size(B, N, V))


def accept_compact(logits: torch.Tensor, node_tok: torch.Tensor, parent: torch.Tensor, n_nodes: torch.Tensor,
                   kv: torch.Tensor, cache_off: torch.Tensor, cache_len: torch.Tensor, cache_cap: torch.Tensor,
                   n_layers: int = 1, layer_stride_rows: int = 0, out: Optional[dict] = None,
                   workspace: Optional[torch.Tensor] = None, stream=None) -> dict:
    """ddt_accept_compact. logits [B, N, V] f32/bf16; kv pool [rows, row_elems]
    f32/bf16 compacted in place; cache_len [B] i32 advanced in place.
    Returns am, acc_len, acc_nodes, out_tok, bonus, status tensors."""
    B, N, V = logits.shape
    _check(logits, "logits", (torch.float32, torch.bfloat16))
    _check(node_tok, "node_tok", torch.int32, (B, N))
    _check(parent, "parent", torch.int32, (B, N))
    _check(n_nodes, "n_nodes", torch.int32, (B,))
    _check(kv, "kv", (torch.float32, torch.bfloat16))
    _check(cache_off, "cache_off", torch.int64, (B,))
    _check(cache_len, "cache_len", torch.int32, (B,))
    _check(cache_cap, "cache_cap", torch.int32, (B,))
    dev = logits.device
    if out is None:
        out = alloc_accept(B, N, dev)
    _check_out(out, _accept_out_spec(B, N))
    need = accept_compact_workspace_size(B, N, V)
    if workspace is None:
        workspace = torch.zeros(max(need, 256), dtype=torch.uint8, device=dev)  # arrival counters start at 0
    _check(workspace, "workspace", None)
    row_elems = kv.shape[-1]
    with _device(logits, node_tok, parent, n_nodes, kv, cache_off, cache_len, cache_cap,
                 workspace, *out.values(), stream=stream):
        st = load().ddt_accept_compact(_ptr(logits), _dt(logits), V, _ptr(node_tok), _ptr(parent), _ptr(n_nodes),
                                       B, N, _ptr(kv), kv.numel() // row_elems, _dt(kv), row_elems, n_layers,
                                       layer_stride_rows,
                                       _ptr(cache_off), _ptr(cache_len), _ptr(cache_cap), _ptr(out["am"]),
                                       _ptr(out["acc_len"]), _ptr(out["acc_nodes"]), _ptr(out["out_tok"]),
                                       _ptr(out["bonus"]), _ptr(out["status"]), _ptr(workspace),
                                       workspace.numel() * workspace.element_size(), _stream(stream))
    _raise("ddt_accept_compact", st)
    return out


def _accept_out_spec(B: int, N: int) -> dict:
    i32 = torch.int32
    return {"am": (i32, (B, N)), "acc_len": (i32, (B,)), "acc_nodes": (i32, (B, N)), "out_tok": (i32, (B, N)),
            "bonus": (i32, (B,)), "status": (i32, (B,))}


def alloc_accept(B: int, N: int, device) -> dict:
    i32 = dict(dtype=torch.int32, device=device)
    return {"am": torch.empty(B, N, **i32), "acc_len": torch.empty(B, **i32),
            "acc_nodes": torch.empty(B, N, **i32), "out_tok": torch.empty(B, N, **i32),
            "bonus": torch.empty(B, **i32), "status": torch.empty(B, **i32)}


def accept_compact_noalloc(logits: torch.Tensor, node_tok: torch.Tensor, parent: torch.Tensor,
                           n_nodes: torch.Tensor, kv: torch.Tensor, cache_off: torch.Tensor, cache_len: torch.Tensor,
                           cache_cap: torch.Tensor, n_layers: int = 1, layer_stride_rows: int = 0,
                           out: Optional[dict] = None, stream=None) -> dict:
    """ddt_accept_compact_noalloc: the same step as accept_compact, for callers
    that cannot allocate device memory; its scratch is a fixed array inside
    libddt.so (shared by all calls, so calls must not overlap on the GPU)."""
    B, N, V = logits.shape
    _check(logits, "logits", (torch.float32, torch.bfloat16))
    _check(node_tok, "node_tok", torch.int32, (B, N))
    _check(parent, "parent", torch.int32, (B, N))
    _check(n_nodes, "n_nodes", torch.int32, (B,))
    _check(kv, "kv", (torch.float32, torch.bfloat16))
    _check(cache_off, "cache_off", torch.int64, (B,))
    _check(cache_len, "cache_len", torch.int32, (B,))
    _check(cache_cap, "cache_cap", torch.int32, (B,))
    if out is None:
        out = alloc_accept(B, N, logits.device)
    _check_out(out, _accept_out_spec(B, N))
    with _device(logits, node_tok, parent, n_nodes, kv, cache_off, cache_len, cache_cap,
                 *out.values(), stream=stream):
        st = load().ddt_accept_compact_noalloc(_ptr(logits), _dt(logits), V, _ptr(node_tok), _ptr(parent),
                                               _ptr(n_nodes), B, N, _ptr(kv), kv.numel() // kv.shape[-1], _dt(kv),
                                               kv.shape[-1], n_layers,
                                               layer_stride_rows, _ptr(cache_off), _ptr(cache_len),
                                               _ptr(cache_cap), _ptr(out["am"]), _ptr(out["acc_len"]),
                                               _ptr(out["acc_nodes"]), _ptr(out["out_tok"]), _ptr(out["bonus"]),
                                               _ptr(out["status"]), _stream(stream))
    _raise("ddt_accept_compact_noalloc", st)
    return out


def accept_compact_lmhead(hidden: torch.Tensor, w_vocab: torch.Tensor, node_tok: torch.Tensor, parent: torch.Tensor,
                          n_nodes: torch.Tensor, kv: torch.Tensor, cache_off: torch.Tensor, cache_len: torch.Tensor,
                          cache_cap: torch.Tensor, n_layers: int = 1, layer_stride_rows: int = 0,
                          out: Optional[dict] = None, workspace: Optional[torch.Tensor] = None, stream=None) -> dict:
    """ddt_accept_compact_lmhead: accept_compact with the target's LM head
    folded into the argmax. hidden [B, N, d] bf16 (the verify rows' final
    hidden states), w_vocab [V, d] bf16; the logits are never materialised.
    Returns the same tensors as accept_compact."""
    B, N, d = hidden.shape
    V = w_vocab.shape[0]
    _check(hidden, "hidden", torch.bfloat16)
    _check(w_vocab, "w_vocab", torch.bfloat16, (V, d))
    _check(node_tok, "node_tok", torch.int32, (B, N))
    _check(parent, "parent", torch.int32, (B, N))
    _check(n_nodes, "n_nodes", torch.int32, (B,))
    _check(kv, "kv", (torch.float32, torch.bfloat16))
    _check(cache_off, "cache_off", torch.int64, (B,))
    _check(cache_len, "cache_len", torch.int32, (B,))
    _check(cache_cap, "cache_cap", torch.int32, (B,))
    dev = hidden.device
    if out is None:
        out = alloc_accept(B, N, dev)
    _check_out(out, _accept_out_spec(B, N))
    need = accept_compact_workspace_size(B, N, V)
    if workspace is None:
        workspace = torch.zeros(max(need, 256), dtype=torch.uint8, device=dev)  # row keys start at 0
    _check(workspace, "workspace", None)
    row_elems = kv.shape[-1]
    with _device(hidden, w_vocab, node_tok, parent, n_nodes, kv, cache_off, cache_len, cache_cap, workspace,
                 *out.values(), stream=stream):
        st = load().ddt_accept_compact_lmhead(
            _ptr(hidden), _ptr(w_vocab), d, V, _ptr(node_tok), _ptr(parent), _ptr(n_nodes), B, N, _ptr(kv),
            kv.numel() // row_elems, _dt(kv), row_elems, n_layers, layer_stride_rows, _ptr(cache_off),
            _ptr(cache_len), _ptr(cache_cap), _ptr(out["am"]), _ptr(out["acc_len"]), _ptr(out["acc_nodes"]),
            _ptr(out["out_tok"]), _ptr(out["bonus"]), _ptr(out["status"]), _ptr(workspace),
            workspace.numel() * workspace.element_size(), _stream(stream))
    _raise("ddt_accept_compact_lmhead", st)
    return out
