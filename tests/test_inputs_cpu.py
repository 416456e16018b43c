"""The seeded input generator keeps the recipe it states: fixed bits per seed,
the stated distributions' support, and packed lengths that hit the total
within their bounds."""
import numpy as np
import pytest
import torch

from gated_deltanet_chunked_rule_b200.inputs import WORKLOADS, Workload, make_inputs, scaled, varlen_lengths


def test_same_seed_same_bits_other_seed_other_bits():
    w = Workload("det", B=2, T=100, Hq=2, Hv=4, K=64, V=64, h0_std=0.02, grads=True, seed=5)
    a, b, c = make_inputs(w), make_inputs(w), make_inputs(scaled(w, seed=6))
    for name in ("q", "k", "v", "g", "beta", "h0", "do", "dht"):
        assert torch.equal(a[name], b[name]), name
        assert not torch.equal(a[name], c[name]), name


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_workload_support_and_shapes(name):
    w = WORKLOADS[name]
    if w.T > 8192:  # the same recipe on a shorter prefix keeps this test quick
        w = scaled(w, T=4096, varlen=None if w.varlen is None else (4, 64, 2048, 4096))
    x = make_inputs(w)
    N = w.B if w.varlen is None else w.varlen[0]
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    assert x["q"].shape == (w.B, w.T, w.Hq, w.K) and x["q"].dtype == dt
    assert x["v"].shape == (w.B, w.T, w.Hv, w.V) and x["v"].dtype == dt
    assert x["g"].dtype == torch.float32 and x["beta"].dtype == torch.float32
    # q, k unit L2 norm per (token, head), up to one bf16 rounding of each element
    for t in ("q", "k"):
        n = x[t].double().norm(dim=-1)
        assert torch.allclose(n, torch.ones_like(n), atol=1e-2 if dt == torch.bfloat16 else 1e-6), t
    g, beta = x["g"].double(), x["beta"].double()
    assert (g < 0).all() and (beta > 0).all() and (beta < 1).all()
    # E[softplus(Z)] for Z ~ N(0, 1) is 0.806; a head-scaled gate multiplies it by
    # e^a with a ~ U(-2, 0) drawn once per value head, so each head's mean gate lies in
    # [-0.806, -0.806 e^-2] (15 % slack for sampling), and the plain gate's is -0.806
    mean = g.mean(dim=(0, 1))
    if w.gate == "headscaled":
        assert (mean >= -0.806 * 1.15).all() and (mean <= -0.806 * np.exp(-2.0) * 0.85).all()
        assert mean.max() - mean.min() > 0.05  # the scale differs between heads
    else:
        assert torch.allclose(mean, torch.full_like(mean, -0.806), atol=0.1)
    if w.h0_std is not None:
        assert x["h0"].shape == (N, w.Hv, w.K, w.V)
        assert abs(x["h0"].double().std().item() - w.h0_std) < 0.1 * w.h0_std
    if w.varlen is not None:
        cu = x["cu_seqlens"].numpy()
        assert cu[0] == 0 and cu[-1] == w.T and np.all(np.diff(cu) >= w.varlen[1])
        assert np.all(np.diff(cu) <= w.varlen[2])


@pytest.mark.parametrize("ns,lo,hi,total", [(16, 64, 8192, 32768), (3, 1, 10, 12), (5, 4, 4, 20)])
def test_varlen_lengths_hit_total_within_bounds(ns, lo, hi, total):
    L = varlen_lengths(np.random.default_rng(0), ns, lo, hi, total)
    assert L.sum() == total and L.min() >= lo and L.max() <= hi and len(L) == ns


def test_unreachable_total_is_refused():
    with pytest.raises(ValueError):
        varlen_lengths(np.random.default_rng(0), 4, 10, 20, 100)
