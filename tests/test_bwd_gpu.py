"""Backward parity on the GPU: gradients from the CUDA path (through the C ABI)
vs the fp64 oracle's hand-derived reverse mode, on the same seeded inputs.
Gate: relative Frobenius error <= 1e-2 per gradient tensor; fp32 problems are
also held to 1e-4 so that a small wrong term cannot hide under bf16 noise."""
import numpy as np
import pytest
import torch

from gated_deltanet_chunked_rule_b200.inputs import WORKLOADS, Workload, make_inputs, scaled
from parity_util import TOL_GRAD_REL, f64, gpu_fwd, rel_fro, to_dev

pytestmark = pytest.mark.gpu
NAMES = ("dq", "dk", "dv", "dbeta", "dg", "dh0")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gated_deltanet_chunked_rule_b200 import build
    build.build()


def gpu_bwd(x, use_saved=True):
    import gated_deltanet_chunked_rule_b200 as gdn
    d = to_dev(x)
    saved = None
    if use_saved:
        _, _, saved = gpu_fwd(x, save_for_backward=True)
    out = gdn.chunk_gated_delta_rule_bwd(
        d["q"], d["k"], d["v"], d["g"], d["beta"], saved, d["do"], d.get("dht"), d["scale"],
        d.get("h0"), d.get("cu_seqlens"), x.get("cu_seqlens"))
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    return dict(zip(NAMES, out))


def oracle_bwd(oracle, x):
    cu = None if x.get("cu_seqlens") is None else x["cu_seqlens"].numpy()
    return oracle.bwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["do"],
                      dht=x.get("dht"), h0=x.get("h0"), cu_seqlens=cu)


def check(oracle, x, g, label, tol=TOL_GRAD_REL):
    r = oracle_bwd(oracle, x)
    errs = {n: rel_fro(f64(g[n]), r[n]) for n in NAMES}
    print(f"[grad parity] {label}: " + "  ".join(f"{n} {e:.2e}" for n, e in errs.items()))
    bad = {n: e for n, e in errs.items() if not e <= tol}
    assert not bad, (label, bad)
    return errs


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("K,V", [(64, 64), (64, 128), (128, 64), (128, 128)])
def test_small_ragged_shapes(oracle_mod, dtype, K, V):
    w = Workload(f"bwd_{dtype}_{K}x{V}", B=2, T=200, Hq=2, Hv=4, K=K, V=V, dtype=dtype,
                 h0_std=0.02, grads=True, seed=K + 2 * V)
    x = make_inputs(w)
    check(oracle_mod, x, gpu_bwd(x), w.name, tol=1e-4 if dtype == "fp32" else TOL_GRAD_REL)


@pytest.mark.parametrize("T", [1, 64, 65])
def test_chunk_boundaries(oracle_mod, T):
    w = Workload(f"bwd_T{T}", B=1, T=T, Hq=1, Hv=1, K=64, V=64, dtype="fp32", h0_std=0.5,
                 grads=True, dht_std=0.5, seed=T)
    x = make_inputs(w)
    check(oracle_mod, x, gpu_bwd(x), w.name, tol=1e-4)


def test_varlen_with_empty_sequences(oracle_mod):
    w = Workload("bwd_varlen", B=1, T=400, Hq=2, Hv=4, K=128, V=128, dtype="fp32", grads=True,
                 seed=11)
    x = make_inputs(w)
    x["cu_seqlens"] = torch.tensor([0, 70, 70, 200, 400], dtype=torch.int32)
    gen = torch.Generator().manual_seed(3)
    x["h0"] = 0.1 * torch.randn((4, 4, 128, 128), generator=gen)
    x["dht"] = 0.1 * torch.randn((4, 4, 128, 128), generator=gen)
    g = gpu_bwd(x)
    check(oracle_mod, x, g, "bwd_varlen", tol=1e-4)
    # empty sequence: dh0 = dht exactly
    torch.testing.assert_close(g["dh0"][1].cpu(), x["dht"][1], rtol=0, atol=0)


def test_saved_equals_recompute():
    w = Workload("bwd_saved", B=1, T=300, Hq=2, Hv=4, K=128, V=128, h0_std=0.02, grads=True,
                 seed=12)
    x = make_inputs(w)
    a = gpu_bwd(x, use_saved=True)
    b = gpu_bwd(x, use_saved=False)
    for n in NAMES:
        torch.testing.assert_close(a[n], b[n], rtol=0, atol=0)


def test_autograd_function(oracle_mod):
    import gated_deltanet_chunked_rule_b200 as gdn
    w = Workload("bwd_autograd", B=1, T=150, Hq=1, Hv=2, K=64, V=64, dtype="fp32",
                 h0_std=0.1, grads=True, seed=13)
    x = make_inputs(w)
    d = to_dev(x)
    leaves = {n: d[n].clone().requires_grad_(True) for n in ("q", "k", "v", "g", "beta", "h0")}
    o, fin = gdn.chunk_gated_delta_rule(leaves["q"], leaves["k"], leaves["v"], leaves["g"],
                                        leaves["beta"], d["scale"], leaves["h0"], True)
    ((o * d["do"]).sum() + (fin * d["dht"]).sum()).backward()
    g = dict(dq=leaves["q"].grad, dk=leaves["k"].grad, dv=leaves["v"].grad,
             dbeta=leaves["beta"].grad, dg=leaves["g"].grad, dh0=leaves["h0"].grad)
    check(oracle_mod, x, g, "bwd_autograd", tol=1e-4)


@pytest.mark.parametrize("name", ["bwd_b2_t4096_h16", "qwen_prefill_t8192_hv32", "long_split_t65536_h8",
                                  "varlen_16seq_32k_h32"])
def test_full_size_workloads(oracle_mod, name):
    w = scaled(WORKLOADS[name], grads=True)
    x = make_inputs(w)
    check(oracle_mod, x, gpu_bwd(x), name)


def test_varlen_bf16_tensor_core_path(oracle_mod):
    # bf16 K = V = 128 runs the tensor-core backward: ragged and empty sequences,
    # per-sequence h0 and dht
    w = Workload("bwd_varlen_bf16", B=1, T=520, Hq=2, Hv=4, K=128, V=128, grads=True, seed=14)
    x = make_inputs(w)
    x["cu_seqlens"] = torch.tensor([0, 0, 130, 137, 137, 520], dtype=torch.int32)
    gen = torch.Generator().manual_seed(5)
    x["h0"] = 0.02 * torch.randn((5, 4, 128, 128), generator=gen)
    x["dht"] = 0.01 * torch.randn((5, 4, 128, 128), generator=gen)
    g = gpu_bwd(x)
    check(oracle_mod, x, g, "bwd_varlen_bf16")
    for n in (0, 3):  # empty sequences: dh0 = dht exactly
        torch.testing.assert_close(g["dh0"][n].cpu(), x["dht"][n], rtol=0, atol=0)


def test_tensor_core_and_cuda_core_backward_agree(oracle_mod, monkeypatch):
    w = Workload("bwd_paths", B=1, T=333, Hq=2, Hv=4, K=128, V=128, h0_std=0.02, grads=True,
                 seed=15)
    x = make_inputs(w)
    a = gpu_bwd(x)
    monkeypatch.setenv("GDN_IMPL", "simt")
    b = gpu_bwd(x)
    monkeypatch.delenv("GDN_IMPL")
    ea = check(oracle_mod, x, a, "bwd tensor-core")
    eb = check(oracle_mod, x, b, "bwd cuda-core")
    for n in NAMES:
        assert rel_fro(f64(a[n]), f64(b[n])) <= TOL_GRAD_REL, n


def test_backward_deterministic():
    w = Workload("bwd_det", B=1, T=700, Hq=2, Hv=4, K=128, V=128, h0_std=0.02, grads=True, seed=16)
    x = make_inputs(w)
    a = gpu_bwd(x)
    b = gpu_bwd(x)
    for n in NAMES:
        torch.testing.assert_close(a[n], b[n], rtol=0, atol=0)


def test_backward_from_states_saved_by_a_split_forward(oracle_mod, monkeypatch):
    # the forward stores every chunk's entry state and Delta in `saved`; with the
    # sequence split the output pass stores them, and the backward reuses them
    w = Workload("bwd_split_saved", B=1, T=1100, Hq=2, Hv=4, K=128, V=128, h0_std=0.02, grads=True,
                 seed=17)
    x = make_inputs(w)
    monkeypatch.setenv("GDN_NSEG", "3")
    g = gpu_bwd(x, use_saved=True)
    monkeypatch.delenv("GDN_NSEG")
    check(oracle_mod, x, g, "bwd from split-forward states")


def _split_inputs(seed):
    # packed batch: an empty sequence, one shorter than the segment count (empty
    # segments), a long one and a ragged tail; per-sequence h0 and dht
    w = Workload("bwd_split", B=1, T=1500, Hq=2, Hv=4, K=128, V=128, grads=True, seed=seed)
    x = make_inputs(w)
    x["cu_seqlens"] = torch.tensor([0, 0, 100, 1037, 1500], dtype=torch.int32)
    gen = torch.Generator().manual_seed(seed + 1)
    x["h0"] = 0.02 * torch.randn((4, 4, 128, 128), generator=gen)
    x["dht"] = 0.01 * torch.randn((4, 4, 128, 128), generator=gen)
    return x


@pytest.mark.parametrize("nseg", [2, 3, 7])
def test_backward_sequence_split_matches_oracle_and_unsplit(oracle_mod, monkeypatch, nseg):
    # Sequence split of the reverse scan: each segment maps the gradient at its end
    # to Q dh + r (Q the transposed product of its chunks' operators); the segments'
    # end gradients are composed backwards from dht, then every segment reruns
    # from its own. The forward runs unsplit, so only the backward differs.
    x = _split_inputs(23)
    monkeypatch.setenv("GDN_NSEG", "1")
    _, _, saved = gpu_fwd(x, save_for_backward=True)
    import gated_deltanet_chunked_rule_b200 as gdn
    d = to_dev(x)

    def bwd():
        out = gdn.chunk_gated_delta_rule_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], saved, d["do"], d["dht"],
                                             d["scale"], d["h0"], d["cu_seqlens"], x["cu_seqlens"])
        torch.cuda.synchronize()
        assert gdn.device_status() == 0
        return dict(zip(NAMES, out))

    g1 = bwd()
    monkeypatch.setenv("GDN_NSEG", str(nseg))
    g2 = bwd()
    monkeypatch.delenv("GDN_NSEG")
    check(oracle_mod, x, g2, f"bwd split{nseg}")
    for n in NAMES:
        assert rel_fro(f64(g2[n]), f64(g1[n])) <= TOL_GRAD_REL, n
    torch.testing.assert_close(g2["dh0"][0].cpu(), x["dht"][0], rtol=0, atol=0)  # empty sequence


def test_backward_sequence_split_slow_decay(oracle_mod, monkeypatch):
    # nearly-undecayed gates: dht reaches dh0 through every segment boundary
    w = Workload("bwd_split_slow", B=1, T=1024, Hq=1, Hv=2, K=128, V=128, h0_std=0.05, grads=True, seed=24)
    x = make_inputs(w)
    x["g"] = x["g"] * 0.01
    x["dht"] = 0.01 * torch.randn((1, 2, 128, 128), generator=torch.Generator().manual_seed(3))
    monkeypatch.setenv("GDN_NSEG", "4")
    g = gpu_bwd(x)
    monkeypatch.delenv("GDN_NSEG")
    check(oracle_mod, x, g, "bwd split slow decay")


@pytest.mark.parametrize("Hq,Hv", [(2, 6), (1, 4), (4, 12)])
def test_larger_head_groups(oracle_mod, Hq, Hv):
    # groups of 3 and 4 value heads per qk head: the per-chunk gradient kernel sums
    # dq and dk over every head of the group on chip (dk accumulated in TMEM by
    # each next head's products, dq parked between heads)
    w = Workload(f"bwd_g{Hv // Hq}", B=1, T=333, Hq=Hq, Hv=Hv, K=128, V=128, h0_std=0.02, grads=True,
                 seed=40 + Hv)
    x = make_inputs(w)
    check(oracle_mod, x, gpu_bwd(x), w.name)


def test_empty_batch_backward():
    # T = 0: no token, so dq, dk, dv, dg, dbeta are empty and dh0 = dht exactly
    import gated_deltanet_chunked_rule_b200 as gdn
    for K, V in ((64, 64), (128, 128)):
        w = Workload("bwd_empty", B=2, T=0, Hq=1, Hv=2, K=K, V=V, h0_std=0.02, grads=True)
        x = to_dev(make_inputs(w))
        _, _, saved = gdn.chunk_gated_delta_rule_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"],
                                                     initial_state=x["h0"], save_for_backward=True)
        out = gdn.chunk_gated_delta_rule_bwd(x["q"], x["k"], x["v"], x["g"], x["beta"], saved, x["do"],
                                             x["dht"], x["scale"], x["h0"])
        torch.cuda.synchronize()
        assert gdn.device_status() == 0
        g = dict(zip(NAMES, out))
        for n in ("dq", "dk", "dv", "dbeta", "dg"):
            assert g[n].numel() == 0
        torch.testing.assert_close(g["dh0"], x["dht"], rtol=0, atol=0)


@pytest.mark.parametrize("name", ["qwen_prefill_t8192_hv32"])
def test_slow_decay_backward_full_size(oracle_mod, name):
    # g x 0.01 at the headline shape: the reverse scan's bf16 operands
    # accumulate over all 128 chunks
    w = scaled(WORKLOADS[name], grads=True)
    x = make_inputs(w)
    x["g"] = x["g"] * 0.01
    check(oracle_mod, x, gpu_bwd(x), name + "_slow")


@pytest.mark.parametrize("use_saved", [True, False])
def test_nonfinite_values_stay_in_their_sequence(use_saved):
    # packed batch whose first sequence ends inside a chunk (100 = 64 + 36): the rest of
    # that chunk's tiles hold the next sequence, here full of Inf and NaN in every per-token
    # input the backward reads (q, k, v, dO, g, beta). The backward zeroes those rows
    # before any product, so the first sequence's gradients are bit-equal to a run whose
    # second sequence is finite (with the forward's saved states, and recomputing them).
    w = Workload("iso_bwd", B=1, T=300, Hq=2, Hv=4, K=128, V=128, grads=True, seed=43)
    x = make_inputs(w)
    x["cu_seqlens"] = torch.tensor([0, 100, 300], dtype=torch.int32)
    gen = torch.Generator().manual_seed(5)
    x["h0"] = 0.02 * torch.randn((2, 4, 128, 128), generator=gen)
    x["dht"] = 0.01 * torch.randn((2, 4, 128, 128), generator=gen)
    ref = gpu_bwd(x, use_saved)
    xb = dict(x)
    for key in ("q", "k", "v", "do"):
        t = x[key].clone()
        t[:, 100:120] = float("inf")
        t[:, 130:140] = float("nan")
        xb[key] = t
    for key in ("g", "beta"):
        t = x[key].clone()
        t[:, 100:140] = float("nan")
        xb[key] = t
    g = gpu_bwd(xb, use_saved)
    for n in ("dq", "dk", "dv", "dbeta", "dg"):
        assert torch.isfinite(g[n][:, :100]).all(), n
        torch.testing.assert_close(g[n][:, :100], ref[n][:, :100], rtol=0, atol=0)
    assert torch.isfinite(g["dh0"][0]).all()
    torch.testing.assert_close(g["dh0"][0], ref["dh0"][0], rtol=0, atol=0)
