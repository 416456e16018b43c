"""gdn_chunk_fwd_noalloc: the forward entry point for callers that cannot
allocate device memory (a plugin whose host engine owns every device
allocation, or a latency-critical path that must not call cudaMalloc/cudaFree,
which can synchronise the device). It takes its scratch from a static device
array inside the library instead of a caller workspace.

Checked here through the C ABI: two calls in a row each match the ordinary
gdn_chunk_fwd (caller workspace) within the forward parity tolerance, and a
problem whose scratch exceeds the static array is refused up front. This file
is collected last so that a stop at the first failure has run everything else.
"""
import ctypes

import pytest
import torch

from gated_deltanet_chunked_rule_b200.inputs import Workload, make_inputs
from parity_util import TOL_BF16_REL, f64, rel_fro, to_dev

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


def test_noalloc_forward_matches_workspace_forward_twice(gdn):
    from gated_deltanet_chunked_rule_b200 import _binding as B
    w = Workload("noalloc", B=1, T=1000, Hq=2, Hv=4, K=128, V=128, h0_std=0.02, seed=21)
    x = to_dev(make_inputs(w))
    o_ref, fin_ref, _ = gdn.chunk_gated_delta_rule_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"],
                                                       x["scale"], initial_state=x["h0"])
    P = gdn.Problem(x["q"], x["v"], x["scale"])
    assert P.fwd_workspace_size() <= B.GDN_NOALLOC_SCRATCH_BYTES
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for _ in range(2):
        o = torch.full_like(o_ref, float("nan"))
        fin = torch.full_like(fin_ref, float("nan"))
        rc = B.lib().gdn_chunk_fwd_noalloc(P.ref(), _p(x["q"]), _p(x["k"]), _p(x["v"]),
                                           _p(x["g"]), _p(x["beta"]), _p(x["h0"]), _p(o), _p(fin),
                                           stream)
        assert rc == B.GDN_OK, B.status_string(rc)
        torch.cuda.synchronize()
        assert gdn.device_status() == 0
        assert rel_fro(f64(o), f64(o_ref)) <= TOL_BF16_REL
        assert rel_fro(f64(fin), f64(fin_ref)) <= TOL_BF16_REL


def test_noalloc_refuses_problems_beyond_the_static_scratch(gdn):
    from gated_deltanet_chunked_rule_b200 import _binding as B
    # T=65536, Hv=8, bf16: Ainv alone needs 1024 chunks * 8 heads * 8 KiB = 64 MiB.
    prob = B.gdn_problem(1, 65536, 8, 8, 128, 128, 0, None, None, B.GDN_DTYPE_BF16, 0.088)
    assert B.lib().gdn_fwd_workspace_size(ctypes.byref(prob)) > B.GDN_NOALLOC_SCRATCH_BYTES
    d = ctypes.c_void_p(1 << 20)
    rc = B.lib().gdn_chunk_fwd_noalloc(ctypes.byref(prob), d, d, d, d, d, None, d, None, None)
    assert rc == B.GDN_ERR_WORKSPACE
