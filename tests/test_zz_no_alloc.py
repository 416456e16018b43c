"""gdn_chunk_fwd_noalloc: the forward entry point for callers that cannot
allocate device memory (a plugin whose host engine owns every device
allocation, or a latency-critical path that must not call cudaMalloc/cudaFree,
which can synchronise the device). It takes its scratch from a static device
array inside the library instead of a caller workspace.

Checked here through the C ABI: two calls in a row each equal, bit for bit,
the ordinary gdn_chunk_fwd run with a caller workspace filled with NaN (the
same kernels on the same inputs, so nothing but stale scratch could make them
differ), with a call on a different, larger problem (other seed, packed
sequences) in between that leaves the shared array full of its own data; a
problem whose scratch exceeds the static array is refused up front. This file
is collected last so that a stop at the first failure has run everything else.
"""
import ctypes

import pytest
import torch

from gated_deltanet_chunked_rule_b200.inputs import Workload, make_inputs
from parity_util import to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gdn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gated_deltanet_chunked_rule_b200 import build
    build.build()
    import gated_deltanet_chunked_rule_b200 as g
    return g


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(gdn, B, x, P, o, fin):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = B.lib().gdn_chunk_fwd_noalloc(P.ref(), _p(x["q"]), _p(x["k"]), _p(x["v"]), _p(x["g"]), _p(x["beta"]),
                                       _p(x.get("h0")), _p(o), _p(fin), stream)
    assert rc == B.GDN_OK, B.status_string(rc)
    torch.cuda.synchronize()
    assert gdn.device_status() == 0


def test_noalloc_forward_equals_workspace_forward_twice(gdn):
    from gated_deltanet_chunked_rule_b200 import _binding as B
    w = Workload("noalloc", B=1, T=1000, Hq=2, Hv=4, K=128, V=128, h0_std=0.02, seed=21)
    x = to_dev(make_inputs(w))
    P = gdn.Problem(x["q"], x["v"], x["scale"])
    assert P.fwd_workspace_size() <= B.GDN_NOALLOC_SCRATCH_BYTES
    ws = torch.full((P.fwd_workspace_size(),), 0xFF, dtype=torch.uint8, device="cuda")  # NaN patterns
    o_ref, fin_ref, _ = gdn.chunk_gated_delta_rule_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"],
                                                       initial_state=x["h0"], workspace=ws)
    # a different problem in between: another seed, packed sequences, more scratch
    w2 = Workload("noalloc_other", B=1, T=1900, Hq=2, Hv=4, K=128, V=128, h0_std=0.05, seed=22)
    x2 = make_inputs(w2)
    x2["cu_seqlens"] = torch.tensor([0, 700, 701, 1900], dtype=torch.int32)
    x2["h0"] = 0.05 * torch.randn((3, 4, 128, 128), generator=torch.Generator().manual_seed(3))
    x2 = to_dev(x2)
    P2 = gdn.Problem(x2["q"], x2["v"], x2["scale"], x2["cu_seqlens"], x2["cu_seqlens"].cpu())
    assert P.fwd_workspace_size() < P2.fwd_workspace_size() <= B.GDN_NOALLOC_SCRATCH_BYTES
    for i in range(2):
        o = torch.full_like(o_ref, float("nan"))
        fin = torch.full_like(fin_ref, float("nan"))
        _noalloc(gdn, B, x, P, o, fin)
        assert torch.equal(o, o_ref) and torch.equal(fin, fin_ref), f"call {i}"
        if i == 0:
            o2 = torch.empty_like(x2["v"])
            f2 = torch.empty((3, 4, 128, 128), dtype=torch.float32, device="cuda")
            _noalloc(gdn, B, x2, P2, o2, f2)
            assert torch.isfinite(o2).all()


def test_noalloc_refuses_problems_beyond_the_static_scratch(gdn):
    from gated_deltanet_chunked_rule_b200 import _binding as B
    # T=65536, Hv=8, bf16: Ainv alone needs 1024 chunks * 8 heads * 8 KiB = 64 MiB.
    prob = B.gdn_problem(1, 65536, 8, 8, 128, 128, 0, None, None, B.GDN_DTYPE_BF16, 0.088)
    assert B.lib().gdn_fwd_workspace_size(ctypes.byref(prob)) > B.GDN_NOALLOC_SCRATCH_BYTES
    d = ctypes.c_void_p(1 << 20)
    rc = B.lib().gdn_chunk_fwd_noalloc(ctypes.byref(prob), d, d, d, d, d, None, d, None, None)
    assert rc == B.GDN_ERR_WORKSPACE
