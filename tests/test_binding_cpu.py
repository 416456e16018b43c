"""Argument checks of the Python binding, on CPU: every tensor whose raw pointer
reaches the library must be a contiguous tensor on q's CUDA device with the
shape and dtype the C ABI expects, because the kernels trust the sizes in
gdn_problem. CPU tensors are refused outright (there is no CPU path)."""
import pytest
import torch

import gated_deltanet_chunked_rule_b200 as gdn
from gated_deltanet_chunked_rule_b200 import api

B, T, Hq, Hv, K, V = 2, 100, 2, 4, 64, 64


def tensors(dtype=torch.bfloat16, N=B):
    return dict(q=torch.zeros(B, T, Hq, K, dtype=dtype), k=torch.zeros(B, T, Hq, K, dtype=dtype),
                v=torch.zeros(B, T, Hv, V, dtype=dtype), g=torch.zeros(B, T, Hv),
                beta=torch.zeros(B, T, Hv), h0=torch.zeros(N, Hv, K, V),
                do=torch.zeros(B, T, Hv, V, dtype=dtype), dht=torch.zeros(N, Hv, K, V))


def check(x, **over):
    x = {**x, **over}
    P = api.Problem(x["q"], x["v"], 0.125)
    api._check_tensors(P, x["q"].device, **x)


def test_cpu_tensors_are_refused_by_every_entry_point():
    x = tensors()
    with pytest.raises(ValueError, match="CUDA"):
        gdn.chunk_gated_delta_rule_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], 0.125, x["h0"])
    with pytest.raises(ValueError, match="CUDA"):
        gdn.chunk_gated_delta_rule_bwd(x["q"], x["k"], x["v"], x["g"], x["beta"], None, x["do"],
                                       x["dht"], 0.125, x["h0"])
    with pytest.raises(ValueError, match="CUDA"):
        gdn.recurrent_gated_delta_rule(x["q"], x["k"], x["v"], x["g"], x["beta"], 0.125, x["h0"])
    with pytest.raises(ValueError, match="CUDA"):
        gdn.chunk_gated_delta_rule(x["q"], x["k"], x["v"], x["g"], x["beta"])


def test_consistent_tensors_pass():
    check(tensors())
    check(tensors(torch.float32))
    check(tensors(), h0=None, dht=None, do=None)


@pytest.mark.parametrize("name,bad,err", [
    ("g", torch.zeros(B, T, Hv, dtype=torch.bfloat16), TypeError),        # gates are fp32
    ("beta", torch.zeros(B, T, Hv + 1), ValueError),                       # wrong head count
    ("k", torch.zeros(B, T, Hq, K), TypeError),                            # k's dtype != q's
    ("v", torch.zeros(B, T - 1, Hv, V, dtype=torch.bfloat16), ValueError),  # v shorter than q
    ("h0", torch.zeros(B + 1, Hv, K, V), ValueError),                      # one state per sequence
    ("h0", torch.zeros(B, Hv, K, V, dtype=torch.float64), TypeError),      # states are fp32
    ("dht", torch.zeros(B, Hv, K * V), ValueError),                        # [N, Hv, K, V]
    ("do", torch.zeros(B, T, Hv, V), TypeError),                           # do in the input dtype
    ("out", torch.zeros(B, T, Hv, V // 2, dtype=torch.bfloat16), ValueError),
    ("final", torch.zeros(B, Hv, K, V).transpose(2, 3), ValueError),        # not contiguous
    ("workspace", torch.zeros(16, dtype=torch.float32), TypeError),         # raw bytes
    ("g", torch.zeros(B, T, Hv, device="meta"), ValueError),                # another device
])
def test_inconsistent_tensor_is_refused(name, bad, err):
    public = {"h0": "initial_state", "final": "final_state"}.get(name, name)
    with pytest.raises(err, match=public):
        check(tensors(), **{name: bad})


def test_short_saved_buffer_is_refused():
    x = tensors()
    P = api.Problem(x["q"], x["v"], 0.125)
    need = P.saved_size()
    api._check_tensors(P, x["q"].device, **x, saved=torch.zeros(need, dtype=torch.uint8))
    with pytest.raises(ValueError, match="saved"):
        api._check_tensors(P, x["q"].device, **x, saved=torch.zeros(need - 1, dtype=torch.uint8))


def test_packed_batch_states_follow_cu_seqlens():
    # with cu_seqlens the batch is packed (B = 1) and there is one state per sequence
    q = torch.zeros(1, 300, Hq, K, dtype=torch.bfloat16)
    v = torch.zeros(1, 300, Hv, V, dtype=torch.bfloat16)
    cu = torch.tensor([0, 100, 100, 300], dtype=torch.int32)
    P = api.Problem(q, v, 0.125, cu, cu)
    assert P.N == 3
    kw = dict(q=q, k=q.clone(), v=v, g=torch.zeros(1, 300, Hv), beta=torch.zeros(1, 300, Hv))
    api._check_tensors(P, q.device, **kw, h0=torch.zeros(3, Hv, K, V))
    with pytest.raises(ValueError, match="initial_state"):
        api._check_tensors(P, q.device, **kw, h0=torch.zeros(1, Hv, K, V))
    with pytest.raises(ValueError, match="cu_seqlens"):
        api.Problem(q, v, 0.125, cu.view(1, -1))
    with pytest.raises(ValueError, match="q and v"):
        api.Problem(q[0], v, 0.125)
