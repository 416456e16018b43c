"""Failure detection on the GPU without a GPU fault.

Every wait inside the library's warp-specialised kernels (on a TMA or
tensor-core completion, or on another warp's hand-over counter) is bounded in
wall-clock time: instead of hanging, it gives up, records GDN_ERR_TIMEOUT in
the per-device status word and lets the kernel return. This checks that path
with the library's own wait helpers on waits that can never be satisfied (an
mbarrier phase nothing completes, a counter nothing publishes) in a kernel
that has nothing else in flight, then that the context is still usable: a
normal forward on the same stream afterwards is bit-equal to one taken before.
"""
import ctypes

import pytest
import torch

from gated_deltanet_chunked_rule_b200.inputs import Workload, make_inputs
from parity_util import gpu_fwd

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gdn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gated_deltanet_chunked_rule_b200 import build
    build.build()
    import gated_deltanet_chunked_rule_b200 as g
    return g


def _selftest(limit_ns):
    from gated_deltanet_chunked_rule_b200 import _binding as B
    elapsed = torch.zeros(2, dtype=torch.int64, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = B.lib().gdn_selftest_wait_timeout(ctypes.c_ulonglong(limit_ns), ctypes.c_void_p(elapsed.data_ptr()), stream)
    assert rc == B.GDN_OK, B.status_string(rc)
    torch.cuda.synchronize()
    return [int(v) for v in elapsed.cpu()]


def test_bounded_waits_give_up_and_report_timeout(gdn):
    w = Workload("after_timeout", B=1, T=300, Hq=2, Hv=4, K=128, V=128, h0_std=0.02, seed=31)
    x = make_inputs(w)
    before = gpu_fwd(x)
    assert gdn.device_status() == 0
    limit = 1_000_000  # 1 ms
    e = _selftest(limit)
    print(f"[timeout] mbarrier wait gave up after {e[0] / 1e6:.3f} ms, counter wait after {e[1] / 1e6:.3f} ms")
    for t in e:
        # neither wait was satisfied, and each gave up soon after its limit
        assert t != -1 and limit <= t < limit + 50_000_000
    assert gdn.device_status() == 5  # GDN_ERR_TIMEOUT
    assert gdn.device_status() == 0  # cleared by the read
    after = gpu_fwd(x)
    torch.testing.assert_close(after[0], before[0], rtol=0, atol=0)
    torch.testing.assert_close(after[1], before[1], rtol=0, atol=0)
    assert gdn.device_status() == 0


def test_kernel_wait_limit_is_two_seconds(gdn):
    # the limit the library's kernels use (limit 0 = that default)
    e = _selftest(0)
    print(f"[timeout] default limit: {e[0] / 1e9:.3f} s (mbarrier), {e[1] / 1e9:.3f} s (counter)")
    for t in e:
        assert 2.0e9 <= t < 2.2e9
    assert gdn.device_status() == 5
