"""ctypes binding of libgdn.so: argument marshalling only.

Every step of the computation runs in the library's CUDA kernels; PyTorch is
used here for device memory (outputs, workspace) and for the current stream.
There is no fallback: if libgdn.so is missing or cannot be loaded, every call
raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libgdn.so")

GDN_OK = 0
GDN_ERR_INVALID_ARG = 1
GDN_ERR_UNSUPPORTED = 2
GDN_ERR_WORKSPACE = 3
GDN_ERR_CUDA = 4
GDN_ERR_TIMEOUT = 5
GDN_ERR_DEVICE_ARG = 6

GDN_DTYPE_F32 = 0
GDN_DTYPE_BF16 = 1

# Every symbol include/gdn.h declares (checked by the CPU tests).
EXPORTS = (
    "gdn_fwd_workspace_size",
    "gdn_bwd_workspace_size",
    "gdn_saved_size",
    "gdn_chunk_fwd",
    "gdn_chunk_bwd",
    "gdn_get_device_status",
    "gdn_status_string",
    "gdn_version",
    "gdn_timing_enable",
    "gdn_timing_report",
    "gdn_chunk_fwd_noalloc",
    "gdn_recurrent_fwd",
    "gdn_selftest_wait_timeout",
)

# Size of the static scratch array behind gdn_chunk_fwd_noalloc.
GDN_NOALLOC_SCRATCH_BYTES = 16 << 20


class gdn_problem(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("T", ctypes.c_int), ("Hq", ctypes.c_int), ("Hv", ctypes.c_int),
        ("K", ctypes.c_int), ("V", ctypes.c_int), ("num_seqs", ctypes.c_int),
        ("cu_seqlens", ctypes.c_void_p), ("cu_seqlens_host", ctypes.c_void_p),
        ("dtype", ctypes.c_int), ("scale", ctypes.c_float),
    ]


class GdnError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        super().__init__(f"{fn} failed: {status_string(code)} ({code})")


_lib = None
_lock = threading.Lock()


def lib() -> ctypes.CDLL:
    """Loads libgdn.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with "
                    "`python -m gated_deltanet_chunked_rule_b200.build` (needs nvcc)")
            L = ctypes.CDLL(LIB_PATH)
            vp, sz, i = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
            pp = ctypes.POINTER(gdn_problem)
            for fn in ("gdn_fwd_workspace_size", "gdn_bwd_workspace_size", "gdn_saved_size"):
                getattr(L, fn).argtypes = [pp]
                getattr(L, fn).restype = sz
            L.gdn_chunk_fwd.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
            L.gdn_chunk_fwd.restype = i
            L.gdn_chunk_bwd.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                        vp, vp, sz, vp]
            L.gdn_chunk_bwd.restype = i
            L.gdn_chunk_fwd_noalloc.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
            L.gdn_chunk_fwd_noalloc.restype = i
            L.gdn_recurrent_fwd.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
            L.gdn_recurrent_fwd.restype = i
            L.gdn_get_device_status.argtypes = [vp]
            L.gdn_get_device_status.restype = i
            L.gdn_status_string.argtypes = [i]
            L.gdn_status_string.restype = ctypes.c_char_p
            L.gdn_timing_enable.argtypes = [i]
            L.gdn_timing_enable.restype = i
            L.gdn_timing_report.argtypes = [ctypes.c_char_p, sz]
            L.gdn_timing_report.restype = i
            L.gdn_selftest_wait_timeout.argtypes = [ctypes.c_ulonglong, vp, vp]
            L.gdn_selftest_wait_timeout.restype = i
            L.gdn_version.argtypes = []
            L.gdn_version.restype = ctypes.c_char_p
            _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().gdn_status_string(int(code)).decode()


def check(fn: str, code: int):
    if code != GDN_OK:
        raise GdnError(fn, code)


def timing_enable(on: bool) -> None:
    check("gdn_timing_enable", lib().gdn_timing_enable(1 if on else 0))


def timing_report() -> dict:
    """{kernel name: (launches, total_ms)} since the last timing_enable(True)."""
    import json
    n = lib().gdn_timing_report(None, 0)
    if n < 0:
        raise GdnError("gdn_timing_report", -n)
    buf = ctypes.create_string_buffer(n + 1)
    lib().gdn_timing_report(buf, n + 1)
    return {k: (int(v[0]), float(v[1])) for k, v in json.loads(buf.value.decode()).items()}
