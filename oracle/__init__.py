"""fp64 CPU oracle for the gated delta rule -- TEST INFRASTRUCTURE ONLY.

This package is the independent checker for the CUDA library. Only the tests,
``__graft_entry__.smoke()`` and the CPU-baseline and reference legs of
``bench.py`` (both time this oracle on the host cores) may import it. It shares no code with the CUDA path and must never be used to produce a
product result.

The arithmetic lives in ``gdn_oracle.c`` (plain C, fp64, token by token):

    S_t = exp(g_t) S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
    o_t = scale * S_t q_t                  state S in R^{V x K}, h = S^T

with the argument list of ``chunk_gated_delta_rule`` /
``chunk_gated_delta_rule_bwd`` in the FlashQLA write-up (page 1, sections
"高级 API 示例" and "底层 API"). This module only marshals numpy arrays to the C
library (compiling it with gcc on first use) and back.

Parity status of each function (pins are in tests/test_oracle_*.py):
  fwd  -- pinned: brute-force dense unrolling, closed forms, invariants,
          linearity, hand-worked golden example.
  bwd  -- pinned: central finite differences and adjoint identities against
          fwd, plus closed-form scalar gradients.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB = os.path.join(_HERE, "libgdn_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile gdn_oracle.c into oracle/libgdn_oracle.so with gcc."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", tmp, _SRC, "-lpthread", "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            dp = ctypes.POINTER(ctypes.c_double)
            ip = ctypes.POINTER(ctypes.c_int32)
            i = ctypes.c_int
            lib.gdn_oracle_fwd.argtypes = [i, i, i, i, i, i, i, ip, dp, dp, dp, dp, dp,
                                           ctypes.c_double, dp, dp, dp, i]
            lib.gdn_oracle_fwd.restype = i
            lib.gdn_oracle_bwd.argtypes = [i, i, i, i, i, i, i, ip, dp, dp, dp, dp, dp,
                                           ctypes.c_double, dp, dp, dp, dp, dp, dp, dp, dp, dp, i]
            lib.gdn_oracle_bwd.restype = i
            _lib = lib
    return _lib


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor: widen exactly (bf16/fp32 -> fp64)
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a, ctype=ctypes.c_double):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _dims(q, v, cu_seqlens):
    B, T, Hq, K = q.shape
    Hv, V = v.shape[2], v.shape[3]
    if cu_seqlens is None:
        return B, T, Hq, Hv, K, V, 0, None, B
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
    return B, T, Hq, Hv, K, V, len(cu) - 1, cu, len(cu) - 1


def fwd(q, k, v, g, beta, scale, h0=None, cu_seqlens=None, nthreads=None):
    """Token-by-token forward in fp64.

    Returns (o [B,T,Hv,V], final_state [N,Hv,K,V]) as float64 numpy arrays.
    """
    q, k, v, g, beta, h0 = (_f64(x) for x in (q, k, v, g, beta, h0))
    B, T, Hq, Hv, K, V, ns, cu, N = _dims(q, v, cu_seqlens)
    o = np.zeros((B, T, Hv, V))
    fin = np.zeros((N, Hv, K, V))
    rc = _load().gdn_oracle_fwd(B, T, Hq, Hv, K, V, ns, _ptr(cu, ctypes.c_int32),
                                _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale),
                                _ptr(h0), _ptr(o), _ptr(fin),
                                int(nthreads or default_threads()))
    if rc != 0:
        raise ValueError(f"gdn_oracle_fwd failed with code {rc}")
    return o, fin


def bwd(q, k, v, g, beta, scale, d_o, dht=None, h0=None, cu_seqlens=None, nthreads=None):
    """Hand-derived reverse mode in fp64.

    Returns dict(dq, dk, dv, dg, dbeta, dh0) as float64 numpy arrays; dq and
    dk are summed over the value heads of each qk-head group, dg is with
    respect to the raw per-token log-decay.
    """
    q, k, v, g, beta, h0, d_o, dht = (_f64(x) for x in (q, k, v, g, beta, h0, d_o, dht))
    B, T, Hq, Hv, K, V, ns, cu, N = _dims(q, v, cu_seqlens)
    out = dict(dq=np.zeros_like(q), dk=np.zeros_like(k), dv=np.zeros((B, T, Hv, V)),
               dg=np.zeros((B, T, Hv)), dbeta=np.zeros((B, T, Hv)), dh0=np.zeros((N, Hv, K, V)))
    rc = _load().gdn_oracle_bwd(B, T, Hq, Hv, K, V, ns, _ptr(cu, ctypes.c_int32),
                                _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale),
                                _ptr(h0), _ptr(d_o), _ptr(dht),
                                _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]),
                                _ptr(out["dg"]), _ptr(out["dbeta"]), _ptr(out["dh0"]),
                                int(nthreads or default_threads()))
    if rc != 0:
        raise ValueError(f"gdn_oracle_bwd failed with code {rc}")
    return out
