"""CPU oracle for the DDTree tree-verify step (test infrastructure only).

Only the test-suite, the smoke check and the benchmark's CPU-baseline leg use
this package; the CUDA library never imports or calls it.
"""
from .ddt_oracle import (  # noqa: F401
    ERR_CAPACITY,
    ERR_INPUT,
    OK,
    accept_compact,
    accept_walk,
    build_tree,
    drafter_topk,
    lmhead_argmax,
    lmhead_f32_error_bound,
    lmhead_logits,
    lmhead_valid_argmax,
    row_argmax,
    verify_attn,
    visible_keys,
    widen,
    widen_logits,
)
