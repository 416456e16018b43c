"""What bench.py divides by a kernel's time.

The roofline of a kernel (kernel_work) counts the method's own work in the rows
of the hot path that kernel implements: the dense contractions of the 64-token
chunked method and the method's inputs and outputs the kernel reads or writes,
no intermediates. The forward's kernels add up to the whole forward of
algorithmic(), the backward's to the whole backward.

The design bytes (kernel_bytes, reported as design_bytes / design_frac) are
the per-unit figures of this design (per token and value head at K = V = 128,
bf16, 64-token chunks, G = Hv / Hq value heads per qk head) times the units
one launch processes, plus the fp32 per-sequence states a kernel touches."""
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


@pytest.mark.parametrize("w", [
    WORKLOADS["qwen_prefill_t8192_hv32"], WORKLOADS["long_split_t65536_h8"],
    WORKLOADS["varlen_16seq_32k_h32"], WORKLOADS["bwd_b2_t4096_h16"],
    Workload("g4", B=2, T=4096, Hq=4, Hv=16, K=128, V=128, h0_std=0.02),
])
def test_kernel_flops_add_up_to_the_chains(w):
    alg = bench.algorithmic(w)
    f = {k: bench.kernel_work(k, w)[0] for k in ("prep3", "fwd_hybrid", "bwd_dh", "bwd_grad")}
    assert f["prep3"] + f["fwd_hybrid"] == alg["f_fwd"]
    assert f["bwd_dh"] + f["bwd_grad"] == alg["f_bwd"]


def test_headline_kernel_work_by_hand():
    w = WORKLOADS["qwen_prefill_t8192_hv32"]
    C, K, V, Hq, Hv, T = 64, 128, 128, 16, 32, 8192
    # per-chunk gradients: Hq*4CK + Hv*(14CK + 8CV + 12KV + 4C^2) per token, 107.4 GFLOP
    F, B = bench.kernel_work("bwd_grad", w)
    assert F == T * (Hq * 4 * C * K + Hv * (14 * C * K + 8 * C * V + 12 * K * V + 4 * C * C))
    assert F == pytest.approx(107.37e9, rel=1e-3)
    # q, k, v, do, g, beta in; dq, dk, dv, dg, dbeta out (bf16 / fp32), no state
    assert B == T * (4 * Hq * K * 2 + 3 * Hv * V * 2 + 4 * Hv * 4)
    # the chain kernel: q, k in, o and the final state out, h0 absent
    F, B = bench.kernel_work("fwd_hybrid", w)
    assert F == T * Hv * (6 * K * V + 2 * C * V)
    assert B == T * (2 * Hq * K * 2 + Hv * V * 2) + Hv * K * V * 4
    # the forward as a whole is bound by HBM at 205.5 MB -> 31.4 us at the measured copy peak
    alg = bench.algorithmic(w)
    assert alg["b_fwd"] == pytest.approx(205.5e6, rel=2e-3)


def test_kernel_roofline_takes_the_binding_side():
    w = WORKLOADS["qwen_prefill_t8192_hv32"]
    pk = {"hbm_gbs": 6539.5, "bf16_tflops": 1606.3}
    F, B = bench.kernel_work("bwd_grad", w)
    r = bench.kernel_roofline("bwd_grad", w, 256.4e-6, pk)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["frac"] == pytest.approx(F / 1606.3e12 / 256.4e-6)
    assert r["achieved"] / r["peak"] == pytest.approx(r["frac"])
    r = bench.kernel_roofline("fwd_hybrid", w, 234e-6, pk)
    assert r["bound"] == "hbm" and r["frac"] == pytest.approx(B and bench.kernel_work("fwd_hybrid", w)[1] / 6539.5e9 / 234e-6)
    assert bench.kernel_roofline("fwd_split_compose", w, 1e-5, pk) is None
