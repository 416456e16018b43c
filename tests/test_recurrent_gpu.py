"""Parity of the token-by-token (decode) step, gdn_recurrent_fwd, on the GPU:
o and the final state vs the fp64 oracle, whose forward is this very
recurrence taken token by token; same tolerances as the chunked forward
(fp32: max-abs 1e-4; bf16: relative Frobenius 5e-3)."""
import pytest
import torch

from gated_deltanet_chunked_rule_b200.inputs import Workload, make_inputs
from parity_util import TOL_BF16_REL, check_fwd, f64, gpu_fwd, rel_fro, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gated_deltanet_chunked_rule_b200 import build
    build.build()


def gpu_rec(x, h0=None, final=None):
    import gated_deltanet_chunked_rule_b200 as gdn
    d = to_dev(x)
    h0 = d.get("h0") if h0 is None else h0
    o, fin = gdn.recurrent_gated_delta_rule(d["q"], d["k"], d["v"], d["g"], d["beta"], d["scale"], h0,
                                            d.get("cu_seqlens"), x.get("cu_seqlens"), final_state=final)
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    return o, fin


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("K,V", [(64, 64), (128, 128), (128, 64)])
@pytest.mark.parametrize("T", [1, 7])
def test_decode_step_matches_oracle(oracle_mod, dtype, K, V, T):
    # a batch of sequences, T tokens each, grouped heads, a nonzero start state
    w = Workload(f"dec_{dtype}_{K}x{V}_T{T}", B=6, T=T, Hq=2, Hv=4, K=K, V=V, dtype=dtype, h0_std=0.05,
                 seed=31 + K + V + T)
    x = make_inputs(w)
    o, fin = gpu_rec(x)
    e = check_fwd(oracle_mod, x, o, fin, w.name)
    print(f"[decode {w.name}] o err {e[0]:.3e} final err {e[1]:.3e}")


def test_decode_varlen_with_empty_sequences(oracle_mod):
    w = Workload("dec_varlen", B=1, T=23, Hq=2, Hv=4, K=128, V=128, seed=37)
    x = make_inputs(w)
    x["cu_seqlens"] = torch.tensor([0, 0, 1, 9, 9, 23], dtype=torch.int32)
    x["h0"] = 0.05 * torch.randn((5, 4, 128, 128), generator=torch.Generator().manual_seed(4))
    o, fin = gpu_rec(x)
    check_fwd(oracle_mod, x, o, fin, "dec_varlen")
    for n in (0, 3):  # empty sequences keep their state exactly
        torch.testing.assert_close(fin[n].cpu(), x["h0"][n], rtol=0, atol=0)


def test_decode_in_place_and_token_by_token_loop():
    # final_state aliasing h0 updates in place; T calls of one token give exactly
    # the state and outputs of one call over T tokens
    w = Workload("dec_loop", B=3, T=5, Hq=2, Hv=4, K=128, V=128, h0_std=0.05, seed=38)
    x = make_inputs(w)
    o_all, fin_all = gpu_rec(x)
    state = to_dev(x)["h0"].clone()
    outs = []
    for t in range(w.T):
        xt = dict(x)
        for name in ("q", "k", "v", "g", "beta"):
            xt[name] = x[name][:, t:t + 1].contiguous()
        o_t, _ = gpu_rec(xt, h0=state, final=state)  # in place
        outs.append(o_t)
    torch.testing.assert_close(state, fin_all, rtol=0, atol=0)
    torch.testing.assert_close(torch.cat(outs, dim=1), o_all, rtol=0, atol=0)


def test_decode_agrees_with_chunked_forward(oracle_mod):
    # several chunks and a ragged tail: the recurrence and the chunked WY form
    w = Workload("dec_vs_chunk", B=2, T=300, Hq=2, Hv=4, K=128, V=128, h0_std=0.05, seed=39)
    x = make_inputs(w)
    o_r, f_r = gpu_rec(x)
    o_c, f_c, _ = gpu_fwd(x)
    check_fwd(oracle_mod, x, o_r, f_r, "dec_vs_chunk recurrent")
    assert rel_fro(f64(o_r), f64(o_c)) <= TOL_BF16_REL and rel_fro(f64(f_r), f64(f_c)) <= TOL_BF16_REL


def test_decode_empty_batch_keeps_state():
    # T = 0: nothing to decode, the state is returned unchanged, bit for bit
    import gated_deltanet_chunked_rule_b200 as gdn
    w = Workload("dec_empty", B=2, T=0, Hq=1, Hv=2, K=128, V=128, h0_std=0.02)
    x = to_dev(make_inputs(w))
    o, fin = gdn.recurrent_gated_delta_rule(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["h0"])
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    assert o.numel() == 0
    torch.testing.assert_close(fin, x["h0"], rtol=0, atol=0)
