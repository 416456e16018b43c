"""The algorithmic bytes bench.py divides by a kernel's time are the per-unit
figures of the design (per token and value head at K = V = 128, bf16, 64-token
chunks, G = Hv / Hq value heads per qk head) times the units one launch
processes, plus the fp32 per-sequence states a kernel touches."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from gated_deltanet_chunked_rule_b200.inputs import WORKLOADS, Workload  # noqa: E402

STATE = 128 * 128 * 4  # one fp32 state per (sequence, value head)


def per_unit(G, saved):
    return {
        "prep3": 512 / G + 1164 + (128 if saved else 0),
        "fwd_hybrid": 512 / G + 1156 + (768 if saved else 0),
        "bwd_recompute": 256 / G + 1540,
        "bwd_dh": 512 / G + 1412,
        "bwd_grad": 1024 / G + 2448,
    }


def states(name, has_h0):
    # per (sequence, value head): which fp32 states the kernel reads or writes
    return {"prep3": 0, "fwd_hybrid": int(has_h0) + 1, "bwd_recompute": int(has_h0),
            "bwd_dh": 2, "bwd_grad": 0}[name]


@pytest.mark.parametrize("w", [
    WORKLOADS["qwen_prefill_t8192_hv32"],                       # G = 2, no h0
    WORKLOADS["long_split_t65536_h8"],                          # G = 1, with h0
    Workload("g4", B=2, T=4096, Hq=4, Hv=16, K=128, V=128, h0_std=0.02),  # G = 4, two rows
])
@pytest.mark.parametrize("saved", [True, False])
def test_kernel_bytes_are_per_unit_figures_times_units(w, saved):
    G = w.Hv // w.Hq
    units = w.B * w.T * w.Hv
    seq_heads = w.B * w.Hv
    for name, b in per_unit(G, saved).items():
        expect = b * units + states(name, w.h0_std is not None) * seq_heads * STATE
        assert bench.kernel_bytes(name, w, saved=saved) == pytest.approx(expect, rel=1e-12), name


def test_headline_gradient_kernel_bytes():
    # 2960 B per token and value head at G = 2: 8192 tokens x 32 heads
    assert bench.kernel_bytes("bwd_grad", WORKLOADS["qwen_prefill_t8192_hv32"], saved=True) == 2960 * 8192 * 32
