"""The C-ABI library builds, loads without a GPU and exports every entry point
include/ddt.h declares; host-side argument checks answer without launching."""
import ctypes
import os
import re

import pytest

from ddtree_speculative_decode_b200 import build, lib

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "ddt.h")


@pytest.fixture(scope="module")
def so():
    build.build()
    return lib.load()


def declared():
    txt = open(HDR).read()
    return re.findall(r"DDT_API\s+[\w\s\*]+?\b(ddt_\w+)\s*\(", txt)


def test_header_declares_the_three_calls():
    names = declared()
    for n in ("ddt_build_tree", "ddt_verify_attn", "ddt_accept_compact"):
        assert n in names


def test_every_declared_symbol_is_exported(so):
    names = declared()
    assert len(names) >= 7
    for n in names:
        assert hasattr(so, n), n
    assert set(names) == set(lib.EXPORTS) | (set(names) - set(lib.EXPORTS))
    for n in lib.EXPORTS:
        assert n in names


def test_status_strings_and_version(so):
    assert lib.status_string(0) == "DDT_OK"
    assert lib.status_string(4) == "DDT_ERR_INPUT"
    assert lib.status_string(99) == "DDT_UNKNOWN_STATUS"
    assert lib.version() >= 100


def _r256(x):
    return (x + 255) // 256 * 256


def _accept_ws(B, N, V):
    """The layout ddt.h documents: a 256-byte status word, then one 8-byte
    running argmax key per row, rounded up to 256 bytes."""
    return 256 + _r256(B * N * 8)


def test_workspace_queries(so):
    assert lib.accept_compact_workspace_size(1, 64, 163840) == _accept_ws(1, 64, 163840) == 256 + 512
    assert lib.accept_compact_workspace_size(65, 8, 16384) == _accept_ws(65, 8, 16384)
    assert lib.accept_compact_workspace_size(64, 256, 163840) < 4 << 20  # fits the no-alloc scratch
    assert lib.accept_compact_workspace_size(0, 64, 10) == 0
    assert so.ddt_verify_attn_workspace_size(1, 8, 4, 64, 16, 32, 0) == 0  # f32 path needs none


def test_host_validation_without_gpu(so):
    # null pointers / out-of-range sizes are rejected before any CUDA call
    st = so.ddt_build_tree(None, None, None, None, 1, 1, 1, 1, None, None, None, None, None, None, None, None, None)
    assert st == lib.DDT_ERR_INVALID_ARG
    p = ctypes.c_void_p(16)
    args = [p] * 4 + [1, 2, 2, 2000] + [p] * 8 + [None]
    assert so.ddt_build_tree(*args) == lib.DDT_ERR_INVALID_ARG
    args = [p] * 4 + [1, 40, 32, 1024] + [p] * 8 + [None]  # 5 bits x 40 levels > 64
    assert so.ddt_build_tree(*args) == lib.DDT_ERR_UNSUPPORTED
    st = so.ddt_verify_attn(p, p, 10, p, p, p, p, 1, 8, 4, 64, 16, ctypes.c_float(-1.0), 32, 0, 0, p, None, None,
                            None, 0, None)
    assert st == lib.DDT_ERR_INVALID_ARG
    st = so.ddt_accept_compact(p, 0, 10, p, p, p, 1, 4, p, 100, 0, 8, 1, 0, p, p, p, p, p, p, p, p, p, p, 0, None)
    assert st == lib.DDT_ERR_INVALID_ARG  # workspace too small
    st = so.ddt_accept_compact(p, 0, 10, p, p, p, 1, 4, p, 0, 0, 8, 1, 0, p, p, p, p, p, p, p, p, p, p, 1 << 20,
                               None)
    assert st == lib.DDT_ERR_INVALID_ARG  # an empty pool


def test_wait_limit_setting(so):
    prev = lib.set_wait_limit_ns(10_000_000)
    try:
        assert prev == 2_000_000_000
        assert lib.set_wait_limit_ns(5) == 10_000_000  # raised to the 1 ms floor
        assert lib.set_wait_limit_ns(0) == 1_000_000   # 0 restores the default
        assert lib.set_wait_limit_ns(0) == 2_000_000_000
    finally:
        lib.set_wait_limit_ns(0)


def test_status_names(so):
    assert lib.status_string(lib.DDT_ERR_TIMEOUT) == "DDT_ERR_TIMEOUT"
    assert lib.status_string(lib.DDT_ERR_BOUNDS) == "DDT_ERR_BOUNDS"


def test_noalloc_accept_rejects_sizes_beyond_its_array(so):
    # 512 x 1024 rows of 8-byte keys + the 256-byte status word > the 4 MiB array:
    # rejected on the host before anything touches the GPU
    p = ctypes.c_void_p(256)
    assert lib.accept_compact_workspace_size(512, 1024, 163840) > 4 << 20
    st = so.ddt_accept_compact_noalloc(p, 1, 163840, p, p, p, 512, 1024, p, 1 << 20, 1, 576, 1, 0, p, p, p, p, p, p,
                                       p, p, p, None)
    assert st == lib.DDT_ERR_UNSUPPORTED
    st = so.ddt_accept_compact_noalloc(None, 1, 163840, p, p, p, 1, 64, p, 1 << 20, 1, 576, 1, 0, p, p, p, p, p, p,
                                       p, p, p, None)
    assert st == lib.DDT_ERR_INVALID_ARG


def test_drafter_topk_host_validation(so):
    p = ctypes.c_void_p(256)
    # nulls, K outside [1, min(V, 32)], bad dtype: rejected before any CUDA call
    assert so.ddt_drafter_topk(None, 1, 100, 4, 8, p, p, None, None) == lib.DDT_ERR_INVALID_ARG
    assert so.ddt_drafter_topk(p, 1, 100, 4, 33, p, p, None, None) == lib.DDT_ERR_INVALID_ARG
    assert so.ddt_drafter_topk(p, 1, 4, 4, 5, p, p, None, None) == lib.DDT_ERR_INVALID_ARG
    assert so.ddt_drafter_topk(p, 1, 100, 4, 0, p, p, None, None) == lib.DDT_ERR_INVALID_ARG
    assert so.ddt_drafter_topk(p, 7, 100, 4, 8, p, p, None, None) == lib.DDT_ERR_INVALID_ARG
    assert so.ddt_drafter_topk(p, 1, 100, 0, 8, p, p, None, None) == lib.DDT_ERR_INVALID_ARG
    # grid and slice arithmetic bounds
    assert so.ddt_drafter_topk(p, 1, 100, 1 << 28, 8, p, p, None, None) == lib.DDT_ERR_UNSUPPORTED
    assert so.ddt_drafter_topk(p, 1, (1 << 30) + 1, 4, 8, p, p, None, None) == lib.DDT_ERR_UNSUPPORTED


def test_one_device_per_call():
    import torch
    a = torch.zeros(2)
    b = torch.zeros(2, device="meta")
    with lib._device(a, a, None):  # one device (and None skipped): nothing to switch
        pass
    with pytest.raises(ValueError):
        lib._device(a, b)


def test_supplied_outputs_are_checked():
    import torch
    with pytest.raises((TypeError, ValueError)):
        lib._check_out({"status": torch.zeros(3, dtype=torch.int32)}, {"status": (torch.int32, (3,))})  # not CUDA
    with pytest.raises(ValueError):
        lib._check_out({}, {"status": (torch.int32, (3,))})  # missing
