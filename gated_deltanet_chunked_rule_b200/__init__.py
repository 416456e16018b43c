"""Gated DeltaNet (gated delta rule) chunked prefill for B200 (sm_100a).

The computation lives in libgdn.so (hand-written CUDA, C ABI in
include/gdn.h); this package is its thin Python binding.
"""
from .api import (  # noqa: F401
    Problem,
    chunk_gated_delta_rule,
    chunk_gated_delta_rule_bwd,
    chunk_gated_delta_rule_fwd,
    device_status,
    recurrent_gated_delta_rule,
)
from ._binding import GdnError, lib  # noqa: F401
