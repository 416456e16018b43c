"""Python entry points over the C ABI (include/gdn.h).

The calls follow the FlashQLA write-up's statement of the operation (page 1,
"高级 API 示例" and "底层 API"):

    o, final_state = chunk_gated_delta_rule(q, k, v, g, beta, scale,
                                            initial_state, output_final_state,
                                            cu_seqlens)
    o, final_state, saved = chunk_gated_delta_rule_fwd(...)
    dq, dk, dv, dbeta, dg, dh0 = chunk_gated_delta_rule_bwd(q, k, v, g, beta,
                                                            saved, do, dht, ...)

Shapes: q, k [B,T,Hq,K]; v [B,T,Hv,V] (bf16 or fp32, all the same dtype);
g (per-token log decay), beta [B,T,Hv] fp32; states [N,Hv,K,V] fp32 with
h = S^T. With cu_seqlens (int32 [N+1]) the batch is packed: B == 1.

This module only marshals arguments: it allocates outputs and the workspace
with torch, passes raw pointers and the current CUDA stream to libgdn.so, and
raises if the library reports an error.
"""
from __future__ import annotations

import ctypes
from typing import Optional

import torch

from . import _binding as _b

_DTYPES = {torch.float32: _b.GDN_DTYPE_F32, torch.bfloat16: _b.GDN_DTYPE_BF16}


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


class Problem:
    """Host-side description of one call (gdn_problem plus the cu_seqlens copies)."""

    def __init__(self, q, v, scale, cu_seqlens=None, cu_seqlens_host=None):
        if q.dim() != 4 or v.dim() != 4:
            raise ValueError(f"q and v must be [B, T, H, D], got {tuple(q.shape)} and {tuple(v.shape)}")
        B, T, Hq, K = q.shape
        Hv, V = v.shape[2], v.shape[3]
        if q.dtype not in _DTYPES:
            raise TypeError(f"unsupported dtype {q.dtype}")
        if cu_seqlens is not None:
            if cu_seqlens.dim() != 1 or cu_seqlens.dtype not in (torch.int32, torch.int64):
                raise ValueError("cu_seqlens must be a 1-D integer tensor")
            if cu_seqlens_host is not None and (cu_seqlens_host.device.type != "cpu"
                                                or cu_seqlens_host.shape != cu_seqlens.shape):
                raise ValueError("cu_seqlens_host must be a CPU copy of cu_seqlens")
        self.cu_dev = None
        self.cu_host = None
        num_seqs = 0
        if cu_seqlens is not None:
            if cu_seqlens_host is None:
                cu_seqlens_host = cu_seqlens.detach().to("cpu")
            self.cu_host = cu_seqlens_host.to(torch.int32).contiguous()
            self.cu_dev = cu_seqlens.to(device=q.device, dtype=torch.int32).contiguous()
            num_seqs = self.cu_host.numel() - 1
        self.N = num_seqs if num_seqs else B
        self.c = _b.gdn_problem(B, T, Hq, Hv, K, V, num_seqs,
                                self.cu_dev.data_ptr() if self.cu_dev is not None else None,
                                self.cu_host.data_ptr() if self.cu_host is not None else None,
                                _DTYPES[q.dtype], float(scale))
        self.shape = (B, T, Hq, Hv, K, V)

    def ref(self):
        return ctypes.byref(self.c)

    def fwd_workspace_size(self) -> int:
        return _b.lib().gdn_fwd_workspace_size(self.ref())

    def bwd_workspace_size(self) -> int:
        return _b.lib().gdn_bwd_workspace_size(self.ref())

    def saved_size(self) -> int:
        return _b.lib().gdn_saved_size(self.ref())


def _c(x):
    return None if x is None else x.contiguous()


def _check(P: Problem, dev, *, q, k, v, g, beta, h0=None, out=None, final=None, do=None, dht=None,
           saved=None, workspace=None):
    """Every tensor the library will read or write through a raw pointer: on the
    CUDA device of q, with the shape and dtype the C ABI expects for this problem.
    The kernels trust these sizes, so nothing else guards against a short buffer."""
    if dev.type != "cuda":
        raise ValueError(f"inputs must be CUDA tensors (got {dev}); the library has no CPU path")
    _check_tensors(P, dev, q=q, k=k, v=v, g=g, beta=beta, h0=h0, out=out, final=final, do=do, dht=dht,
                   saved=saved, workspace=workspace)


def _check_tensors(P: Problem, dev, *, q, k, v, g, beta, h0=None, out=None, final=None, do=None,
                   dht=None, saved=None, workspace=None):
    B, T, Hq, Hv, K, V = P.shape
    state = (P.N, Hv, K, V)
    want = {
        "q": (q, (B, T, Hq, K), q.dtype), "k": (k, (B, T, Hq, K), q.dtype),
        "v": (v, (B, T, Hv, V), q.dtype), "g": (g, (B, T, Hv), torch.float32),
        "beta": (beta, (B, T, Hv), torch.float32), "initial_state": (h0, state, torch.float32),
        "out": (out, (B, T, Hv, V), q.dtype), "final_state": (final, state, torch.float32),
        "do": (do, (B, T, Hv, V), q.dtype), "dht": (dht, state, torch.float32),
        "saved": (saved, None, torch.uint8), "workspace": (workspace, None, torch.uint8),
    }
    for name, (t, shape, dtype) in want.items():
        if t is None:
            continue
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{name} must be a torch.Tensor")
        if t.device != dev:
            raise ValueError(f"{name} is on {t.device}, expected {dev}")
        if t.dtype != dtype:
            raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
        if shape is not None and tuple(t.shape) != shape:
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {shape}")
        if shape is not None and not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if saved is not None and saved.numel() < P.saved_size():
        raise ValueError(f"saved holds {saved.numel()} bytes, the problem needs {P.saved_size()}")


def chunk_gated_delta_rule_fwd(q, k, v, g, beta, scale, initial_state=None,
                               output_final_state=True, cu_seqlens=None, cu_seqlens_host=None,
                               save_for_backward=False, workspace=None, out=None):
    """Forward pass. Returns (o, final_state or None, saved or None).

    `saved` holds the in-chunk cumulative gate and (I + A)^-1 of every chunk
    (the "g, A" of page 1's low-level forward) for chunk_gated_delta_rule_bwd.
    """
    q, k, v, g, beta, h0 = map(_c, (q, k, v, g, beta, initial_state))
    P = Problem(q, v, scale, cu_seqlens, cu_seqlens_host)
    B, T, Hq, Hv, K, V = P.shape
    dev = q.device
    _check(P, dev, q=q, k=k, v=v, g=g, beta=beta, h0=h0, out=out, workspace=workspace)
    o = out if out is not None else torch.empty((B, T, Hv, V), dtype=q.dtype, device=dev)
    fin = torch.empty((P.N, Hv, K, V), dtype=torch.float32, device=dev) if output_final_state else None
    saved = torch.empty(P.saved_size(), dtype=torch.uint8, device=dev) if save_for_backward else None
    ws_bytes = P.fwd_workspace_size()
    if workspace is None or workspace.numel() < ws_bytes:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        rc = _b.lib().gdn_chunk_fwd(P.ref(), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0),
                                    _ptr(o), _ptr(fin), _ptr(saved), _ptr(workspace),
                                    workspace.numel(), _stream(dev))
    _b.check("gdn_chunk_fwd", rc)
    return o, fin, saved


def chunk_gated_delta_rule_bwd(q, k, v, g, beta, saved, do, dht=None, scale=None,
                               initial_state=None, cu_seqlens=None, cu_seqlens_host=None,
                               workspace=None):
    """Backward pass. Returns (dq, dk, dv, dbeta, dg, dh0) in page 1's order
    ("dq, dk, dv, db, dg, dh0"); dg is w.r.t. the raw per-token log decay."""
    if scale is None:
        scale = q.shape[-1] ** -0.5
    q, k, v, g, beta, h0, do, dht = map(_c, (q, k, v, g, beta, initial_state, do, dht))
    P = Problem(q, v, scale, cu_seqlens, cu_seqlens_host)
    B, T, Hq, Hv, K, V = P.shape
    dev = q.device
    _check(P, dev, q=q, k=k, v=v, g=g, beta=beta, h0=h0, do=do, dht=dht, saved=saved, workspace=workspace)
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    dg = torch.empty((B, T, Hv), dtype=torch.float32, device=dev)
    dbeta = torch.empty((B, T, Hv), dtype=torch.float32, device=dev)
    dh0 = torch.empty((P.N, Hv, K, V), dtype=torch.float32, device=dev)
    ws_bytes = P.bwd_workspace_size()
    if workspace is None or workspace.numel() < ws_bytes:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        rc = _b.lib().gdn_chunk_bwd(P.ref(), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0),
                                    _ptr(saved), _ptr(do), _ptr(dht), _ptr(dq), _ptr(dk), _ptr(dv),
                                    _ptr(dg), _ptr(dbeta), _ptr(dh0), _ptr(workspace),
                                    workspace.numel(), _stream(dev))
    _b.check("gdn_chunk_bwd", rc)
    return dq, dk, dv, dbeta, dg, dh0


def recurrent_gated_delta_rule(q, k, v, g, beta, scale=None, initial_state=None, cu_seqlens=None,
                               cu_seqlens_host=None, out=None, final_state=None):
    """Token-by-token (decode) step: the same recurrence as the chunked forward, one
    token after another, for a few tokens per sequence (gdn_recurrent_fwd). Returns
    (o, final_state); `final_state` may be `initial_state` itself (updated in place)."""
    if scale is None:
        scale = q.shape[-1] ** -0.5
    q, k, v, g, beta, h0 = map(_c, (q, k, v, g, beta, initial_state))
    P = Problem(q, v, scale, cu_seqlens, cu_seqlens_host)
    B, T, Hq, Hv, K, V = P.shape
    dev = q.device
    _check(P, dev, q=q, k=k, v=v, g=g, beta=beta, h0=h0, out=out, final=final_state)
    o = out if out is not None else torch.empty((B, T, Hv, V), dtype=q.dtype, device=dev)
    if final_state is None:
        final_state = torch.empty((P.N, Hv, K, V), dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        rc = _b.lib().gdn_recurrent_fwd(P.ref(), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0),
                                        _ptr(o), _ptr(final_state), _stream(dev))
    _b.check("gdn_recurrent_fwd", rc)
    return o, final_state


class _ChunkGDN(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, g, beta, scale, h0, output_final_state, cu_seqlens, cu_host):
        o, fin, saved = chunk_gated_delta_rule_fwd(q, k, v, g, beta, scale, h0, output_final_state,
                                                   cu_seqlens, cu_host, save_for_backward=True)
        ctx.save_for_backward(q, k, v, g, beta, h0, saved, cu_seqlens, cu_host)
        ctx.scale = scale
        return o, fin

    @staticmethod
    def backward(ctx, do, dht):
        q, k, v, g, beta, h0, saved, cu, cu_host = ctx.saved_tensors
        dq, dk, dv, dbeta, dg, dh0 = chunk_gated_delta_rule_bwd(
            q, k, v, g, beta, saved, do, dht, ctx.scale, h0, cu, cu_host)
        return dq, dk, dv, dg, dbeta, None, (dh0 if h0 is not None else None), None, None, None


def chunk_gated_delta_rule(q, k, v, g, beta, scale=None, initial_state=None,
                           output_final_state=False, cu_seqlens=None, cu_seqlens_host=None):
    """High-level call: (o, final_state or None), differentiable w.r.t. q, k,
    v, g, beta and initial_state."""
    if scale is None:
        scale = q.shape[-1] ** -0.5
    if cu_seqlens is not None and cu_seqlens_host is None:
        cu_seqlens_host = cu_seqlens.detach().to("cpu")
    if torch.is_grad_enabled() and any(
            t is not None and t.requires_grad for t in (q, k, v, g, beta, initial_state)):
        return _ChunkGDN.apply(q, k, v, g, beta, scale, initial_state, output_final_state,
                               cu_seqlens, cu_seqlens_host)
    o, fin, _ = chunk_gated_delta_rule_fwd(q, k, v, g, beta, scale, initial_state,
                                           output_final_state, cu_seqlens, cu_seqlens_host)
    return o, fin


def device_status(device=None) -> int:
    """Synchronises the current stream and returns/clears the device status word."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    return _b.lib().gdn_get_device_status(_stream(dev))
