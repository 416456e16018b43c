"""Seeded synthetic inputs for the gated delta rule chunked prefill.

This module only draws random numbers and shapes them; it holds none of the
recurrence's arithmetic. Both the CUDA path (tests, bench, smoke) and the fp64
oracle take their inputs from here, so both sides see identical bits.

Recipe (one numpy PCG64 generator per call, ``default_rng(seed)``):

* draw order: [varlen lengths], q, k, v, g-noise, a (per head), beta-noise,
  h0, do, dht -- a tensor that a workload does not use is not drawn;
* every tensor is drawn in fp32; q and k are L2-normalised over K per
  (token, head); the bf16 workloads then round q, k, v, do to bf16
  (round-to-nearest-even, once), g, beta and all states stay fp32;
* g = -softplus(N(0,1)) ("softplus" gate) or g = -exp(a) * softplus(N(0,1))
  with a ~ U(-2, 0) drawn once per value head ("headscaled" gate);
* beta = sigmoid(N(0,1));  h0 ~ N(0, h0_std) (std, not variance);
* do ~ N(0,1), dht ~ N(0, dht_std).

The shapes are those of Qwen-style GDN layers (K = V = 128, v heads grouped
over shared q/k heads), long prefill, variable-length packed batches, and the
small per-GPU head counts left after tensor-parallel sharding, as the FlashQLA
write-up describes its benchmark grid (page 1, "性能基准测试": head counts
{64,48,32,24,16,8} for TP1..TP8). No public dataset is involved.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace
from typing import Optional

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    Hq: int
    Hv: int
    K: int
    V: int
    dtype: str = "bf16"            # dtype of q, k, v (and o, do, dq, dk, dv)
    gate: str = "headscaled"       # "softplus" | "headscaled"
    h0_std: Optional[float] = None  # None -> no initial state
    varlen: Optional[tuple] = None  # (num_seqs, min_len, max_len, total) -> cu_seqlens
    grads: bool = False            # also draw do, dht
    dht_std: float = 0.01
    seed: int = 0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.K)


# The five workloads of the contract (names describe what they are).
WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", B=1, T=256, Hq=2, Hv=2, K=64, V=64, dtype="fp32",
                          gate="softplus"),
    "qwen_prefill_t8192_hv32": Workload("qwen_prefill_t8192_hv32", B=1, T=8192, Hq=16, Hv=32,
                                        K=128, V=128),
    "long_split_t65536_h8": Workload("long_split_t65536_h8", B=1, T=65536, Hq=8, Hv=8, K=128,
                                     V=128, h0_std=0.02),
    "varlen_16seq_32k_h32": Workload("varlen_16seq_32k_h32", B=1, T=32768, Hq=32, Hv=32, K=128,
                                     V=128, h0_std=0.02, varlen=(16, 64, 8192, 32768)),
    "bwd_b2_t4096_h16": Workload("bwd_b2_t4096_h16", B=2, T=4096, Hq=16, Hv=16, K=128, V=128,
                                 grads=True),
}


def varlen_lengths(rng: np.random.Generator, num_seqs: int, lo: int, hi: int, total: int):
    """Lengths log-uniform in [lo, hi], rescaled to sum exactly to ``total``.

    Draw L_i = exp(U(ln lo, ln hi)), rescale so the sum is ``total``, round,
    clip to [lo, hi], then hand the rounding residue out one token at a time,
    longest sequence first, without leaving [lo, hi].
    """
    if num_seqs * lo > total or num_seqs * hi < total:
        raise ValueError("total not reachable with these bounds")
    raw = np.exp(rng.uniform(math.log(lo), math.log(hi), size=num_seqs))
    L = np.clip(np.rint(raw * (total / raw.sum())), lo, hi).astype(np.int64)
    order = np.argsort(-L, kind="stable")
    i = 0
    while L.sum() != total:
        j = order[i % num_seqs]
        step = 1 if L.sum() < total else -1
        if lo <= L[j] + step <= hi:
            L[j] += step
        i += 1
    return L


def _bf16(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)


def _l2norm(x: np.ndarray) -> np.ndarray:
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True, dtype=np.float32))


def _softplus(x: np.ndarray) -> np.ndarray:
    return np.logaddexp(np.float32(0), x).astype(np.float32)


def make_inputs(w: Workload) -> dict:
    """Draw one workload's inputs as CPU torch tensors.

    Returns a dict with q, k [B,T,Hq,K]; v [B,T,Hv,V] (bf16 or fp32); g, beta
    [B,T,Hv] fp32; scale (float); h0 [N,Hv,K,V] fp32 or None; cu_seqlens
    int32 [N+1] or None; and, for gradient workloads, do [B,T,Hv,V] and dht
    [N,Hv,K,V].
    """
    rng = np.random.default_rng(w.seed)
    cu = None
    N = w.B
    if w.varlen is not None:
        ns, lo, hi, total = w.varlen
        if w.B != 1 or w.T != total:
            raise ValueError("varlen workloads pack into B=1, T=total")
        L = varlen_lengths(rng, ns, lo, hi, total)
        cu = np.concatenate([[0], np.cumsum(L)]).astype(np.int32)
        N = ns
    shp_qk = (w.B, w.T, w.Hq, w.K)
    shp_v = (w.B, w.T, w.Hv, w.V)
    q = _l2norm(rng.standard_normal(shp_qk, dtype=np.float32))
    k = _l2norm(rng.standard_normal(shp_qk, dtype=np.float32))
    v = rng.standard_normal(shp_v, dtype=np.float32)
    gn = rng.standard_normal((w.B, w.T, w.Hv), dtype=np.float32)
    if w.gate == "softplus":
        g = -_softplus(gn)
    elif w.gate == "headscaled":
        a = rng.uniform(-2.0, 0.0, size=(w.Hv,)).astype(np.float32)
        g = (-np.exp(a)[None, None, :] * _softplus(gn)).astype(np.float32)
    else:
        raise ValueError(w.gate)
    bn = rng.standard_normal((w.B, w.T, w.Hv), dtype=np.float32)
    beta = (1.0 / (1.0 + np.exp(-bn))).astype(np.float32)
    h0 = None
    if w.h0_std is not None:
        h0 = (w.h0_std * rng.standard_normal((N, w.Hv, w.K, w.V), dtype=np.float32)).astype(np.float32)
    out = dict(scale=w.scale, cu_seqlens=None if cu is None else torch.from_numpy(cu))
    if w.dtype == "bf16":
        out.update(q=_bf16(q), k=_bf16(k), v=_bf16(v))
    elif w.dtype == "fp32":
        out.update(q=torch.from_numpy(q), k=torch.from_numpy(k), v=torch.from_numpy(v))
    else:
        raise ValueError(w.dtype)
    out.update(g=torch.from_numpy(np.ascontiguousarray(g)),
               beta=torch.from_numpy(np.ascontiguousarray(beta)),
               h0=None if h0 is None else torch.from_numpy(h0))
    if w.grads:
        do = rng.standard_normal(shp_v, dtype=np.float32)
        dht = (w.dht_std * rng.standard_normal((N, w.Hv, w.K, w.V), dtype=np.float32)).astype(np.float32)
        out["do"] = _bf16(do) if w.dtype == "bf16" else torch.from_numpy(do)
        out["dht"] = torch.from_numpy(dht)
    return out


def scaled(w: Workload, **kw) -> Workload:
    """A copy of a workload with some fields replaced (smaller test sizes)."""
    return replace(w, **kw)
