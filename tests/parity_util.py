"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
(python binding) and the fp64 oracle on the same seeded inputs, and compare.

Tolerances (written here, used by every parity test):
  fp32 inputs: max-abs error <= 1e-4 on o and final states;
  bf16 inputs with fp32 state: relative Frobenius error <= 5e-3 on o and on
  the final states (all sequences), <= 1e-2 on each gradient.
"""
import numpy as np
import torch

TOL_FP32_MAXABS = 1e-4
TOL_BF16_REL = 5e-3
TOL_GRAD_REL = 1e-2


def to_dev(x, dev="cuda"):
    return {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


def rel_fro(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = np.linalg.norm(b.ravel())
    return float(np.linalg.norm((a - b).ravel()) / (den if den > 0 else 1.0))


def max_abs(a, b):
    return float(np.max(np.abs(np.asarray(a, np.float64) - np.asarray(b, np.float64)))) if np.size(a) else 0.0


def f64(t):
    return t.detach().to("cpu").double().numpy()


def gpu_fwd(x, **kw):
    import gated_deltanet_chunked_rule_b200 as gdn
    d = to_dev(x)
    o, fin, saved = gdn.chunk_gated_delta_rule_fwd(
        d["q"], d["k"], d["v"], d["g"], d["beta"], d["scale"], initial_state=d.get("h0"),
        output_final_state=True, cu_seqlens=d.get("cu_seqlens"),
        cu_seqlens_host=x.get("cu_seqlens"), **kw)
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    return o, fin, saved


def oracle_fwd(oracle, x):
    return oracle.fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], h0=x.get("h0"),
                      cu_seqlens=None if x.get("cu_seqlens") is None else x["cu_seqlens"].numpy())


def check_fwd(oracle, x, o, fin, label=""):
    o_ref, fin_ref = oracle_fwd(oracle, x)
    if x["q"].dtype == torch.float32:
        eo, ef = max_abs(f64(o), o_ref), max_abs(f64(fin), fin_ref)
        assert eo <= TOL_FP32_MAXABS and ef <= TOL_FP32_MAXABS, (label, eo, ef)
    else:
        eo, ef = rel_fro(f64(o), o_ref), rel_fro(f64(fin), fin_ref)
        assert eo <= TOL_BF16_REL and ef <= TOL_BF16_REL, (label, eo, ef)
    return eo, ef
