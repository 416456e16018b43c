"""Chunk-prep kernels checked through their own outputs (the saved buffer):
gamma must be the in-chunk cumulative sum of g, and Ainv must invert
I + A with A_rs = beta_r exp(gamma_r - gamma_s) k_r.k_s (s < r), rebuilt here
in fp64 from the inputs. The residual bound is the rounding of the stored
Ainv: fp32 (CUDA-core prep) or bf16 (tensor-core prep)."""
import numpy as np
import pytest
import torch

from gated_deltanet_chunked_rule_b200.inputs import Workload, make_inputs
from parity_util import gpu_fwd

pytestmark = pytest.mark.gpu


def unpack_saved(saved, x, cu=None):
    B, T, Hq, K = x["q"].shape
    Hv = x["v"].shape[2]
    ntok = B * T
    gbytes = (ntok * Hv * 4 + 255) // 256 * 256
    raw = saved.cpu()
    gamma = raw[: ntok * Hv * 4].view(torch.float32).view(ntok, Hv).double().numpy()
    if cu is None:
        starts = [(b * T + c, min(64, T - c)) for b in range(B) for c in range(0, T, 64)]
    else:
        starts = [(a + c, min(64, b - a - c)) for a, b in zip(cu[:-1], cu[1:]) for c in range(0, b - a, 64)]
    nc = len(starts)
    esz = 4 if x["q"].dtype == torch.float32 else 2
    ab = raw[gbytes: gbytes + nc * Hv * 64 * 64 * esz]
    ainv = (ab.view(torch.float32) if esz == 4 else ab.view(torch.bfloat16)).view(nc, Hv, 64, 64)
    return gamma, ainv.double().numpy(), starts


def check_prep(x, saved, cu=None, tol=None):
    gamma, ainv, starts = unpack_saved(saved, x, cu)
    Hq, Hv = x["q"].shape[2], x["v"].shape[2]
    G = Hv // Hq
    k = x["k"].double().numpy().reshape(-1, Hq, x["k"].shape[-1])
    g = x["g"].double().numpy().reshape(-1, Hv)
    beta = x["beta"].double().numpy().reshape(-1, Hv)
    worst_res, worst_gam = 0.0, 0.0
    for c, (t0, L) in enumerate(starts):
        for h in range(Hv):
            gam_ref = np.cumsum(g[t0:t0 + L, h])
            worst_gam = max(worst_gam, float(np.max(np.abs(gamma[t0:t0 + L, h] - gam_ref))))
            kk = k[t0:t0 + L, h // G]
            gm = gamma[t0:t0 + L, h]
            A = np.tril(beta[t0:t0 + L, h, None] * np.exp(gm[:, None] - gm[None, :]) * (kk @ kk.T), -1)
            X = ainv[c, h, :L, :L]
            res = np.abs((np.eye(L) + A) @ X - np.eye(L)).max()
            worst_res = max(worst_res, float(res))
            # padded part of the stored 64x64 block is the identity
            if L < 64:
                assert np.allclose(ainv[c, h, L:, L:], np.eye(64 - L))
    return worst_gam, worst_res


@pytest.mark.parametrize("impl", ["default", "simt"])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_prep_outputs_invert_the_chunk_matrix(impl, dtype, monkeypatch):
    if impl == "simt":
        monkeypatch.setenv("GDN_IMPL", "simt")
    w = Workload("prep", B=1, T=300, Hq=2, Hv=4, K=128, V=128, dtype=dtype, seed=31)
    x = make_inputs(w)
    _, _, saved = gpu_fwd(x, save_for_backward=True)
    wg, wr = check_prep(x, saved)
    print(f"[prep {impl} {dtype}] gamma err {wg:.2e}  residual {wr:.2e}")
    assert wg <= 1e-5
    assert wr <= (1e-5 if dtype == "fp32" else 2e-2)


def test_prep_varlen_ragged():
    w = Workload("prep_varlen", B=1, T=500, Hq=1, Hv=2, K=128, V=128, seed=32)
    x = make_inputs(w)
    cu = [0, 37, 37, 200, 500]
    x["cu_seqlens"] = torch.tensor(cu, dtype=torch.int32)
    _, _, saved = gpu_fwd(x, save_for_backward=True)
    wg, wr = check_prep(x, saved, cu)
    print(f"[prep varlen] gamma err {wg:.2e}  residual {wr:.2e}")
    assert wg <= 1e-5 and wr <= 2e-2
