"""Benchmark of the gated delta rule chunked prefill on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--fwd-only]

One step = one pass of the whole hot path over one batch of the synthetic
workload: the chunked forward (prep + state propagation/output) followed by
the chunked backward, all in libgdn.so's kernels. The default workload is the
Qwen-style GDN prefill shape B=1, T=8192, Hq=16, Hv=32, K=V=128, bf16 q/k/v,
fp32 gates and state. With N GPUs (torchrun) every rank runs its own copy of
the workload (independent sequences: no collective on the data path) and the
value is all ranks' tokens over the slowest rank's device time.

Prints one JSON line (rank 0). `--impl reference` times the fp64 CPU oracle
(the only reference this method has) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GDN chunk-prefill fwd/bwd Mtokens/s and % of roofline (T=8192, Hv=32, K=V=128)"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
CHUNK = 64


def peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def algorithmic(w, tokens_per_seq=None):
    """Algorithmic flops and bytes of one forward and one backward pass.

    Bytes: inputs read once plus outputs written once. Flops: the dense
    contractions of the 64-token chunked method, counting the q/k Gram
    matrices once per qk head.
      fwd per token: Hq*4CK + Hv*(2CK + 4CV + 6KV)
      bwd per token: Hq*4CK + Hv*(14CK + 10CV + 18KV + 4C^2)
    """
    C, K, V, Hq, Hv = CHUNK, w.K, w.V, w.Hq, w.Hv
    ntok = w.B * w.T
    N = w.varlen[0] if w.varlen else w.B
    e = 2 if w.dtype == "bf16" else 4
    f_fwd = ntok * (Hq * 4 * C * K + Hv * (2 * C * K + 4 * C * V + 6 * K * V))
    f_bwd = ntok * (Hq * 4 * C * K + Hv * (14 * C * K + 10 * C * V + 18 * K * V + 4 * C * C))
    qk = 2 * ntok * Hq * K * e
    vv = ntok * Hv * V * e
    gb = 2 * ntok * Hv * 4
    st = N * Hv * K * V * 4
    h0 = st if w.h0_std is not None else 0
    b_fwd = qk + vv + gb + h0 + vv + st                       # q,k,v,g,beta,h0 -> o, final
    # q,k,v,g,beta,h0,do,dht -> dq,dk,dv,dg,dbeta,dh0
    b_bwd = (qk + vv + gb + h0 + vv + st) + (qk + vv + gb + st)
    return dict(f_fwd=f_fwd, f_bwd=f_bwd, b_fwd=b_fwd, b_bwd=b_bwd, tokens=ntok)


def kernel_work(name, w):
    """Algorithmic work of one launch of a named kernel, by the rows of the hot
    path it implements: (flops of the method's dense contractions in those
    rows, bytes of the method's own inputs and outputs the kernel reads or
    writes). Intermediates of this design (w, u, P, gamma, Ainv, chunk states,
    Delta, dh', dDelta) are not counted: they are design bytes (kernel_bytes).

    Flops per token (C = 64), split from the chain totals of algorithmic():
      prep3 (gamma, A, Ainv, w, u):      Hq*4CK + Hv*(2CK + 2CV)
      fwd_hybrid (chain + output):       Hv*(6KV + 2CV)
      bwd_dh (reverse state scan):       Hv*(2CV + 6KV)
      bwd_grad (per-chunk gradients):    Hq*4CK + Hv*(14CK + 8CV + 12KV + 4C^2)
    so prep3 + fwd_hybrid = the forward and bwd_dh + bwd_grad = the backward.
    Bytes: q, k [T,Hq,K], v, o, do, dv [T,Hv,V] in the input dtype, g, beta,
    dg, dbeta [T,Hv] fp32, states h0, final, dht, dh0 [N,Hv,K,V] fp32, each
    counted once for every kernel that touches it.
    Returns None for a kernel without a row of its own (split composition,
    recompute, plan)."""
    C, K, V, Hq, Hv = CHUNK, w.K, w.V, w.Hq, w.Hv
    ntok = w.B * w.T
    N = w.varlen[0] if w.varlen else w.B
    e = 2 if w.dtype == "bf16" else 4
    qk1 = ntok * Hq * K * e        # q or k (or dq, dk)
    v1 = ntok * Hv * V * e         # v, o, do or dv
    g1 = ntok * Hv * 4             # g, beta, dg or dbeta
    st = N * Hv * K * V * 4        # one state per (sequence, value head)
    h0 = st if w.h0_std is not None else 0
    f_prep = ntok * (Hq * 4 * C * K + Hv * (2 * C * K + 2 * C * V))
    f_chain = ntok * Hv * (6 * K * V + 2 * C * V)
    f_dh = ntok * Hv * (2 * C * V + 6 * K * V)
    f_grad = ntok * (Hq * 4 * C * K + Hv * (14 * C * K + 8 * C * V + 12 * K * V + 4 * C * C))
    table = {
        "prep3": (f_prep, 2 * qk1 + v1 + 2 * g1),                    # q, k, v, g, beta
        "fwd_hybrid": (f_chain, 2 * qk1 + h0 + v1 + st),             # q, k, h0 -> o, final
        "bwd_dh": (f_dh, 2 * qk1 + v1 + st + st),                    # q, k, do, dht -> dh0
        "bwd_grad": (f_grad, 2 * qk1 + 2 * v1 + 2 * g1 + 2 * qk1 + v1 + 2 * g1),
        # q, k, v, do, g, beta -> dq, dk, dv, dg, dbeta
        "recurrent": (ntok * Hv * 8 * K * V, 2 * qk1 + v1 + 2 * g1 + h0 + v1 + st),
    }
    return table.get(name)


def kernel_roofline(name, w, avg_s, pk):
    """The roofline of one kernel on its own rows: time bound = max(F / tensor
    peak, B / HBM peak); the binding side's achieved rate over its peak."""
    work = kernel_work(name, w)
    if work is None or not avg_s:
        return None
    F, B = work
    t_tc = F / (pk["bf16_tflops"] * 1e12)
    t_hbm = B / (pk["hbm_gbs"] * 1e9)
    if t_tc >= t_hbm:
        return {"bound": "tensor", "unit": "TFLOP/s", "achieved": F / avg_s / 1e12,
                "peak": pk["bf16_tflops"], "frac": t_tc / avg_s, "algorithmic_flops": F,
                "algorithmic_bytes": B}
    return {"bound": "hbm", "unit": "GB/s", "achieved": B / avg_s / 1e9, "peak": pk["hbm_gbs"],
            "frac": t_hbm / avg_s, "algorithmic_flops": F, "algorithmic_bytes": B}


def kernel_bytes(name, w, saved=False):
    """Design bytes of one launch of a named kernel: the tensors that kernel
    must read once and write once in this design, intermediates between the
    kernels of the chain included (w, u, P, chunk states, ...). Their ratio to
    the launch time is a streaming efficiency, reported as design_frac beside
    the roofline of kernel_work().

    Per token and value head at K = V = 128, bf16 (e = 2), G = Hv / Hq:
      prep3            2K*e/G (q, k) + V*e (v) + 3*4 (g, beta, gamma) + K*2 (w) + V*4 (u) + C*2 (P)
                       [+ C*e Ainv when saved]
      fwd_hybrid       2K*e/G (q, k) + K*2 (w) + V*4 (u) + C*2 (P) + 4 (gamma) + V*e (o)
                       [+ K*V*e/C (entry states) + V*e (Delta) when saved]
      bwd_recompute    K*e/G (k) + K*2 + V*4 + 4 + K*V*e/C (entry states) + V*e (Delta)
      bwd_dh           2K*e/G (q, k) + K*2 (w) + C*2 (P) + V*e (dO) + 4 + K*V*e/C (dh') + V*e (dDelta)
      bwd_grad         2K*e/G + 2V*e (v, dO) + 8 (gamma, beta) + C*e (Ainv) + 2K*V*e/C (h, dh')
                       + 2V*e (Delta, dDelta) + 2K*e/G (dq, dk, summed over the group on chip)
                       + V*e (dv) + 8 (dg, dbeta)
    plus the per-sequence states (h0, final, dht, dh0: K*V*4 each) where a kernel touches them.
    Entry states, Delta and dDelta are stored per chunk (64 rows, ragged ones padded).
    """
    C, K, V, Hq, Hv = CHUNK, w.K, w.V, w.Hq, w.Hv
    ntok = w.B * w.T
    N = w.varlen[0] if w.varlen else w.B
    e = 2 if w.dtype == "bf16" else 4
    nc = math.ceil(w.T / C) * w.B if not w.varlen else ntok // C + N  # upper bound for packed input
    qk1 = ntok * Hq * K * e
    v1 = ntok * Hv * V * e
    gam = ntok * Hv * 4
    ainv = nc * Hv * C * C * e
    st = N * Hv * K * V * 4
    h0 = st if w.h0_std is not None else 0
    hc = nc * Hv * K * V * 2
    dsb = nc * C * Hv * V * 2   # Delta and dDelta, per chunk
    wb = ntok * Hv * K * 2      # w (bf16)
    ub = ntok * Hv * V * 4      # u (fp32)
    pb = nc * Hv * C * C * 2    # P (bf16)
    prep3 = 2 * qk1 + v1 + 2 * gam + gam + wb + ub + pb
    table = {
        "prep_simt": qk1 + 2 * gam + gam + ainv,               # k, g, beta -> gamma, Ainv
        "prep_tc": qk1 + 2 * gam + gam + ainv,
        "prep3": prep3 + (ainv if saved else 0),                # q,k,v,g,beta -> gamma,w,u,P[,Ainv]
        "fwd_simt": 2 * qk1 + v1 + 2 * gam + ainv + h0 + v1 + st,  # q,k,v,gamma,beta,Ainv,h0 -> o,final
        # q,k,w,u,P,gamma,h0 -> o,final[,entry states,Delta]
        "fwd_hybrid": 2 * qk1 + wb + ub + pb + gam + h0 + v1 + st + ((hc + dsb) if saved else 0),
        "bwd_prep3": prep3 + (0 if saved else ainv),
        "bwd_recompute": qk1 + wb + ub + gam + h0 + hc + dsb,
        "bwd_dh": 2 * qk1 + wb + pb + v1 + gam + st + hc + dsb + st,
        "bwd_grad": 2 * qk1 + 2 * v1 + 2 * gam + ainv + 2 * hc + 2 * dsb + 2 * qk1 + v1 + 2 * gam,
    }
    return table.get(name)


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum, bytes per launch)
# of one ncu capture per kernel (summaries under profiles/), valid only for the
# workload and step they were taken on and only while the kernel's sources are
# byte-identical to the captured build (sha256 over the listed files).
NCU_TRAFFIC = {
    "bwd_grad": dict(workload="qwen_prefill_t8192_hv32", step="fwd+bwd", bytes=639716096 + 118936320,
               sources=["gdn_bwd_grad.cu"],
               sha256="cbba0dec59861f9a29b8689f21bf3da92f4ad43f5d64565573c5b558ed9005f1"),
    "bwd_dh": dict(workload="qwen_prefill_t8192_hv32", step="fwd+bwd", bytes=238085376 + 163700992,
               sources=["gdn_bwd_dh.cu"],
               sha256="5a6cd00f77d5ef975c74a2dd1a54451b37353939ae3b16825381feefd4ebd379"),
    "fwd_hybrid": dict(workload="qwen_prefill_t8192_hv32", step="fwd+bwd", bytes=303272960 + 229458944,
               sources=["gdn_fwd3.cu"],
               sha256="4ab2d3258a8acfdbe40dd99c74f8e65bf27fc06b7a8ca712f094ffff60d52952"),
    "prep3": dict(workload="qwen_prefill_t8192_hv32", step="fwd+bwd", bytes=186969600 + 213129728,
               sources=["gdn_prep3.cu"],
               sha256="819efa9638fb9f2e4f6b742e8ce3fa0267571cb8821d0db411dbdbeae9f90202"),
    "recurrent": dict(workload="decode_b256_hv32", step="decode", bytes=549415168 + 481711104,
               sources=["gdn_recurrent.cu"],
               sha256="35e113de4eda5533922853cf613728b9b8d8c372c9964fd87946edc0413bf6a2"),
}
TRAFFIC_COMMON_SOURCES = ["gdn_internal.cuh", "gdn_warp.cuh", "sm100_ptx.cuh"]


def measured_traffic(kernel, workload, step):
    """ncu DRAM bytes per launch for this kernel, or None if not captured for this
    workload and step or if the kernel's sources changed since the capture."""
    rec = NCU_TRAFFIC.get(kernel)
    if not rec or rec["workload"] != workload or rec["step"] != step:
        return None
    import hashlib
    csrc = os.path.join(os.path.dirname(os.path.abspath(__file__)), "gated_deltanet_chunked_rule_b200", "csrc")
    h = hashlib.sha256()
    try:
        for f in rec["sources"] + TRAFFIC_COMMON_SOURCES:
            with open(os.path.join(csrc, f), "rb") as fh:
                h.update(fh.read())
    except OSError:
        return None
    return rec["bytes"] if h.hexdigest() == rec["sha256"] else None


class Clocks:
    """Samples SM clocks and throttle reasons with nvidia-smi while running."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = os.path.join("/tmp", f"gdn_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f,
                stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


def rank_workload(w, rank):
    """Each rank runs its own independent batch (weak scaling, no collective on the
    data path): the workload's shape, its seed offset by the rank."""
    from gated_deltanet_chunked_rule_b200.inputs import scaled
    return scaled(w, seed=w.seed + rank, grads=True)


def max_over_ranks(x, dist=None, device="cpu"):
    """x on this rank -> its maximum over all ranks (x itself with one rank)."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def slowest_ms(total_ms, dist=None, device="cpu"):
    """The job's time: the slowest rank's device time (max over ranks)."""
    return max_over_ranks(total_ms, dist, device)


def job_mtokens_s(tokens_per_rank, world, steps, total_ms):
    """Whole-job throughput: every rank's tokens over the slowest rank's time."""
    return tokens_per_rank * world * steps / (total_ms * 1e-3) / 1e6


def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def run_reference(args, w):
    """fp64 CPU oracle timed on the host cores on a bounded sample of the workload."""
    import oracle
    from gated_deltanet_chunked_rule_b200.inputs import make_inputs, scaled
    ws, rank, _ = dist_setup()
    if rank != 0:
        return 0
    sample_T = min(w.T, args.ref_tokens)
    ws_ = scaled(w, T=sample_T, varlen=None)
    x = make_inputs(scaled(ws_, grads=True))
    cores = oracle.default_threads()
    oracle.build()

    def step():
        oracle.fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], h0=x["h0"])
        if not args.fwd_only:
            oracle.bwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["do"],
                       dht=x["dht"], h0=x["h0"])

    for _ in range(args.warmup):
        step()
    times = []
    for _ in range(args.steps):
        t = time.perf_counter()
        step()
        times.append(time.perf_counter() - t)
    tok = ws_.B * ws_.T
    ms = 1e3 * statistics.mean(times)
    value = tok / (ms * 1e-3) / 1e6
    sample = (f"first {sample_T} tokens of each of B={w.B} rows, all {w.Hv} heads; "
              f"{'fwd' if args.fwd_only else 'fwd+bwd'} per step")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "Mtokens/s",
        "n_gpus": ws, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        # the same workload as the CUDA arm's line; each step times a bounded sample of
        # it (cpu_baseline.sample), and the value is the sample's tokens over its time
        "config": {"workload": w.name, "B": w.B, "T": w.T, "Hq": w.Hq, "Hv": w.Hv,
                   "K": w.K, "V": w.V, "chunk": CHUNK, "step": "fwd" if args.fwd_only else "fwd+bwd"},
        "cpu_baseline": {"value": value, "unit": "Mtokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "Mtokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def cpu_baseline(args, w):
    """The oracle, as it stands, on this host's CPU cores (bounded sample)."""
    import oracle
    from gated_deltanet_chunked_rule_b200.inputs import make_inputs, scaled
    oracle.build()
    sample_T = min(w.T, args.ref_tokens)
    ws_ = scaled(w, T=sample_T, varlen=None, grads=True)
    x = make_inputs(ws_)
    t = time.perf_counter()
    oracle.fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], h0=x["h0"])
    if not args.fwd_only:
        oracle.bwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["do"], dht=x["dht"],
                   h0=x["h0"])
    dt = time.perf_counter() - t
    tok = ws_.B * ws_.T
    return {"value": tok / dt / 1e6, "unit": "Mtokens/s", "cores": oracle.default_threads(),
            "kind": "oracle",
            "sample": f"one {'fwd' if args.fwd_only else 'fwd+bwd'} pass over the first "
                      f"{sample_T} tokens, all {w.Hv} heads ({dt:.2f} s wall)"}


def run_decode(args):
    """Token-by-token (decode) step through gdn_recurrent_fwd: one token for each of
    B sequences and Hv heads per step, state updated in place. The state (B*Hv*K*V
    fp32, 512 MB here) is larger than L2, so every step moves it from and to HBM;
    the roofline is that traffic against the measured copy bandwidth."""
    import torch
    import gated_deltanet_chunked_rule_b200 as gdn
    gdn.lib()  # fail loudly if the extension is missing
    B, Hq, Hv, K, V = 256, 16, 32, 128, 128
    dev = torch.device("cuda", 0)
    gen = torch.Generator(device=dev).manual_seed(0)
    nrm = torch.nn.functional.normalize
    q = nrm(torch.randn(B, 1, Hq, K, device=dev, generator=gen), dim=-1).bfloat16()
    k = nrm(torch.randn(B, 1, Hq, K, device=dev, generator=gen), dim=-1).bfloat16()
    v = torch.randn(B, 1, Hv, V, device=dev, generator=gen).bfloat16()
    g = -torch.nn.functional.softplus(torch.randn(B, 1, Hv, device=dev, generator=gen))
    beta = torch.sigmoid(torch.randn(B, 1, Hv, device=dev, generator=gen))
    state = 0.02 * torch.randn(B, Hv, K, V, device=dev, generator=gen)
    o = torch.empty(B, 1, Hv, V, device=dev, dtype=torch.bfloat16)

    def step():
        gdn.recurrent_gated_delta_rule(q, k, v, g, beta, None, state, out=o, final_state=state)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with Clocks(0) as clk:
        e0.record()
        for _ in range(args.steps):
            step()
        e1.record()
        torch.cuda.synchronize()
    if gdn.device_status() != 0:
        raise SystemExit("decode step reported a device error")
    ms = e0.elapsed_time(e1) / args.steps
    traffic = 2 * B * Hv * K * V * 4 + B * (2 * Hq * K + 2 * Hv * V) * 2 + 2 * B * Hv * 4
    pk, pk_kind = peaks()
    achieved = traffic / (ms * 1e-3) / 1e9
    print(json.dumps({
        "metric": "GDN decode step Mtokens/s (one token per sequence, state in HBM)",
        "value": B / (ms * 1e3), "unit": "Mtokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "decode_b256_hv32", "B": B, "T": 1, "Hq": Hq, "Hv": Hv, "K": K, "V": V,
                   "step": "decode", "l2": "state 512 MB > L2, updated in place every step"},
        "roofline": {"kernel": "recurrent", "bound": "hbm", "unit": "GB/s", "achieved": achieved,
                     "peak": pk["hbm_gbs"], "peak_kind": f"{pk_kind} hbm_gbs (burst copy)",
                     "traffic": measured_traffic("recurrent", "decode_b256_hv32", "decode"),
                     "algorithmic_bytes": traffic, "frac": achieved / pk["hbm_gbs"]},
        "gpu_launches": args.steps, "clocks": clk.summary()}))


def torchrun_cmd(nproc, argv, port):
    """The command that relaunches this script with one process per GPU."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={nproc}",
            "--master-addr=127.0.0.1", f"--master-port={port}", os.path.abspath(__file__), *argv]


def relaunch(args, argv):
    """`--gpus N` (N > 1) without a torchrun environment: start N local ranks under
    torch.distributed.run and return their exit status. Refuses when fewer than N
    devices are visible (the CPU self-test of the launcher needs none)."""
    import socket
    if not args.dist_selftest:
        import torch
        have = torch.cuda.device_count()
        if have < args.gpus:
            raise SystemExit(f"--gpus {args.gpus}: only {have} CUDA device(s) visible")
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    env = dict(os.environ)
    env.pop("WORLD_SIZE", None)
    return subprocess.call(["timeout", "-k", "60", "1800", *torchrun_cmd(args.gpus, argv, port)], env=env)


def run_dist_selftest(args):
    """Host-side multi-rank path without a GPU (gloo): every rank reports a
    different per-rank time; rank 0 prints the line with the job's max-over-ranks
    time and all ranks' tokens. Used by the CPU test of the `--gpus N` launcher."""
    import datetime
    import torch.distributed as dist
    world, rank, local = dist_setup()
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    mine = 1.0 + rank
    total = slowest_ms(mine, dist, "cpu")
    if rank == 0:
        print(json.dumps({"metric": METRIC, "n_gpus": world, "selftest": True, "ms_per_step": total,
                          "value": job_mtokens_s(1024, world, 1, total)}), flush=True)
    dist.barrier()
    dist.destroy_process_group()
    return 0


def measure(w, steps, warmup, dev, rank, dist=None, timing=True, infer=True):
    """Times fwd (+bwd) steps of one workload on this rank's GPU: CUDA events on
    the launch stream, L2 flushed between steps (outside the events), the max
    over ranks. Returns per-step times, per-kernel times and the chain rooflines."""
    import torch
    import gated_deltanet_chunked_rule_b200 as gdn
    from gated_deltanet_chunked_rule_b200 import _binding
    from gated_deltanet_chunked_rule_b200.inputs import make_inputs

    wr = rank_workload(w, rank)
    xh = make_inputs(wr)
    x = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in xh.items()}
    cu_host = xh["cu_seqlens"]
    P = gdn.Problem(x["q"], x["v"], x["scale"], x["cu_seqlens"], cu_host)
    ws_f = torch.empty(max(P.fwd_workspace_size(), 1), dtype=torch.uint8, device=dev)
    ws_b = torch.empty(max(P.bwd_workspace_size(), 1), dtype=torch.uint8, device=dev)
    o = torch.empty_like(x["v"])
    do_bwd = True
    try:
        _, _, sv = gdn.chunk_gated_delta_rule_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"],
                                                  x["scale"], x["h0"], True, x["cu_seqlens"],
                                                  cu_host, save_for_backward=True)
        gdn.chunk_gated_delta_rule_bwd(x["q"], x["k"], x["v"], x["g"], x["beta"], sv, x["do"],
                                       x["dht"], x["scale"], x["h0"], x["cu_seqlens"], cu_host)
    except _binding.GdnError as e:
        if e.code != _binding.GDN_ERR_UNSUPPORTED:
            raise
        do_bwd = False

    def step(inp, train=True, out=None):
        save = do_bwd and train
        o_, fin_, sv_ = gdn.chunk_gated_delta_rule_fwd(
            inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["scale"], inp["h0"], True,
            inp["cu_seqlens"], cu_host, save_for_backward=save, workspace=ws_f, out=o if out is None else out)
        if save:
            grads = gdn.chunk_gated_delta_rule_bwd(
                inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], sv_, inp["do"], inp["dht"],
                inp["scale"], inp["h0"], inp["cu_seqlens"], cu_host, workspace=ws_b)
            return o_, fin_, grads
        return o_, fin_, None

    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(max(2 * l2, 1 << 20) // 4, dtype=torch.float32, device=dev)

    def timed_steps(n, fn):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(n)]
        for a, b in ev:
            flush.fill_(1.0)
            a.record()
            fn()
            b.record()
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in ev]

    def kernel_pass(fn):
        # the same steps again with the library's event timing on (events on the
        # launch stream around every launch)
        _binding.timing_enable(True)
        timed_steps(steps, fn)
        rep = _binding.timing_report()
        _binding.timing_enable(False)
        return rep

    for _ in range(warmup):
        step(x)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    res = {"x": x, "xh": xh, "step": step, "timed_steps": timed_steps, "do_bwd": do_bwd}
    res["ms_list"] = timed_steps(steps, lambda: step(x))
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    res["total_ms"] = slowest_ms(sum(res["ms_list"]), dist, dev)
    pk, _ = peaks()
    alg = algorithmic(w)

    def chain(F, Bt, ms):
        t_tc = F / (pk["bf16_tflops"] * 1e12)
        t_hbm = Bt / (pk["hbm_gbs"] * 1e9)
        return {"ms": ms, "Mtokens_s": alg["tokens"] / (ms * 1e-3) / 1e6 if ms else None,
                "tflops": F / (ms * 1e-3) / 1e12 if ms else None,
                "gbs": Bt / (ms * 1e-3) / 1e9 if ms else None,
                "bound_us": 1e6 * max(t_tc, t_hbm), "binding": "tensor" if t_tc > t_hbm else "hbm",
                "frac": (1e3 * max(t_tc, t_hbm)) / ms if ms else None}

    if timing:
        rep = kernel_pass(lambda: step(x))
        res["rep"] = rep
        fwd_ms = sum(v[1] for k, v in rep.items() if not k.startswith("bwd")) / steps
        bwd_ms = sum(v[1] for k, v in rep.items() if k.startswith("bwd")) / steps
        res["fwd"] = chain(alg["f_fwd"], alg["b_fwd"], fwd_ms)
        res["bwd"] = chain(alg["f_bwd"], alg["b_bwd"], bwd_ms) if do_bwd else None
    if infer:
        # the plain (inference) forward: nothing saved for a backward
        inf_ms = timed_steps(steps, lambda: step(x, train=False))
        inf_total = slowest_ms(sum(inf_ms), dist, dev)
        res["fwd_infer"] = chain(alg["f_fwd"], alg["b_fwd"], inf_total / steps)
        if timing:
            rep_i = kernel_pass(lambda: step(x, train=False))
            res["rep_infer"] = rep_i
            res["fwd_infer"]["kernels_us"] = {k: 1e3 * v[1] / v[0] for k, v in rep_i.items()}
    res["alg"] = alg
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1,
                    help="GPUs in the job: N replicas, one process per GPU (relaunched under "
                         "torch.distributed.run when not already started by it)")
    ap.add_argument("--steps", type=int, default=20, help="timed steps")
    ap.add_argument("--warmup", type=int, default=5, help="untimed warm-up steps (at least 3)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"],
                    help="reference: time the fp64 oracle on the host cores on a bounded sample")
    ap.add_argument("--workload", default="qwen_prefill_t8192_hv32",
                    help="one of the named synthetic workloads (inputs.py)")
    ap.add_argument("--fwd-only", action="store_true", help="time the forward alone")
    ap.add_argument("--ref-tokens", type=int, default=1024,
                    help="tokens per row in the oracle's bounded sample")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle timing")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the long-sequence and packed-batch workloads of the headline run")
    ap.add_argument("--decode", action="store_true", help="time the token-by-token step instead")
    ap.add_argument("--heads", default=None, help="HQ,HV: override the workload's head counts (sweeps)")
    ap.add_argument("--dist-selftest", action="store_true", help=argparse.SUPPRESS)
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    world, rank, local = dist_setup()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        return relaunch(args, sys.argv[1:])
    if "WORLD_SIZE" in os.environ and world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    if args.dist_selftest:
        return run_dist_selftest(args)
    if args.decode:
        return run_decode(args)

    from gated_deltanet_chunked_rule_b200.inputs import WORKLOADS
    w = WORKLOADS[args.workload]
    if args.heads:
        from dataclasses import replace
        hq, hv = (int(x) for x in args.heads.split(","))
        w = replace(w, name=f"{w.name}_hq{hq}_hv{hv}", Hq=hq, Hv=hv)
    if args.impl == "reference":
        return run_reference(args, w)

    import torch
    import gated_deltanet_chunked_rule_b200 as gdn

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    gdn.lib()  # fail loudly if the extension is missing

    with Clocks(local) as clk:
        r = measure(w, args.steps, args.warmup, dev, rank, dist)
    if args.fwd_only:
        # forward-only line: the plain (inference) forward is the step
        r["total_ms"] = r["fwd_infer"]["ms"] * args.steps
        r["do_bwd"] = False
        r["rep"] = r["rep_infer"]
    do_bwd = r["do_bwd"]
    rep, alg = r["rep"], r["alg"]
    fwd_blocks = (None if args.fwd_only else r["fwd"], r["bwd"] if do_bwd else None, r["fwd_infer"])
    tokens = alg["tokens"]
    total_ms = r["total_ms"]
    ms_step = total_ms / args.steps
    value = job_mtokens_s(tokens, world, args.steps, total_ms)

    kern_total = sum(v[1] for v in rep.values())
    pk, pk_kind = peaks()
    kernels = {}
    for k, v in rep.items():
        avg_s = v[1] / v[0] * 1e-3
        kr = kernel_roofline(k, w, avg_s, pk)
        kernels[k] = {"launches": v[0], "avg_us": 1e3 * v[1] / v[0],
                      "share": v[1] / kern_total if kern_total else None,
                      "frac": kr["frac"] if kr else None, "bound": kr["bound"] if kr else None}
    # the roofline block: the kernel with the largest share of the step's device
    # time among those that implement rows of the hot path, on its own rows
    dom = max((k for k in rep if kernel_work(k, w)), key=lambda k: rep[k][1])
    dom_avg_s = rep[dom][1] / rep[dom][0] * 1e-3
    roofline = {"kernel": dom, **kernel_roofline(dom, w, dom_avg_s, pk)}
    roofline["peak_kind"] = (f"{pk_kind} bf16_tflops (burst)" if roofline["bound"] == "tensor"
                             else f"{pk_kind} hbm_gbs (burst copy)")
    roofline["traffic"] = measured_traffic(dom, w.name, "fwd+bwd" if do_bwd else "fwd")
    db = kernel_bytes(dom, w, saved=do_bwd)
    if db:
        roofline["design_bytes"] = db
        roofline["design_frac"] = db / dom_avg_s / 1e9 / pk["hbm_gbs"]

    # End to end through the public API with host buffers: every step copies its inputs
    # in from pinned host memory and all of its results (o, the final state and, for a
    # training step, every gradient) out to pinned host memory, inside the timed region.
    # The copies are pipelined the way a data loader would run them: step i+1's inputs
    # go in on one stream and step i-1's results come out on another while step i
    # computes (two buffer sets), so the step rate is bound by the larger PCIe
    # direction rather than by the sum of both directions and the compute.
    x, xh, step = r["x"], r["xh"], r["step"]
    names_in = ["q", "k", "v", "g", "beta"] + (["h0"] if xh["h0"] is not None else []) + \
        (["do", "dht"] if do_bwd else [])
    host_in = {k: xh[k].pin_memory() for k in names_in}
    dev_in = [{k: torch.empty_like(x[k]) for k in names_in} for _ in range(2)]
    o_buf = [torch.empty_like(x["v"]) for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    host_out = [{}, {}]
    comp = torch.cuda.current_stream(dev)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    in_ready = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]

    def e2e_run(n):
        t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        t_start.record(s_in)
        for i in range(n):
            b = i & 1
            if i >= 2:
                s_in.wait_event(comp_done[b])  # step i-2 has finished reading buffer set b
            with torch.cuda.stream(s_in):
                for k in names_in:
                    dev_in[b][k].copy_(host_in[k], non_blocking=True)
                in_ready[b].record(s_in)
            comp.wait_event(in_ready[b])
            if i >= 2:
                comp.wait_event(out_done[b])  # step i-2's o has been copied out of o_buf[b]
            inp = dict(x)
            inp.update(dev_in[b])
            o_, fin_, grads = step(inp, train=do_bwd, out=o_buf[b])
            comp_done[b].record(comp)
            outs = [o_, fin_] + (list(grads) if grads is not None else [])
            s_out.wait_event(comp_done[b])
            with torch.cuda.stream(s_out):
                for j, t in enumerate(outs):
                    if j not in host_out[b]:
                        host_out[b][j] = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
                    host_out[b][j].copy_(t, non_blocking=True)
                    t.record_stream(s_out)
                out_done[b].record(s_out)
        t_end.record(s_out)  # the last copy out follows every earlier copy and step
        torch.cuda.synchronize()
        return t_start.elapsed_time(t_end)

    e2e_run(2)
    if dist:
        dist.barrier()
    e2e_total = slowest_ms(e2e_run(args.steps), dist, dev)
    d2h = sum(t.numel() * t.element_size() for t in host_out[0].values())
    e2e = {"value": job_mtokens_s(tokens, world, args.steps, e2e_total), "unit": "Mtokens/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "pipelined": "step i+1's inputs in and step i-1's results out while step i computes "
                        "(three streams, two buffer sets)"}
    del r

    # the long-sequence (sequence split) and packed-batch workloads, at their full
    # sizes: per-step fwd / bwd chains and their rooflines
    extra = {}
    if not args.no_extra and not args.heads and w.name == "qwen_prefill_t8192_hv32":
        for name in ("long_split_t65536_h8", "varlen_16seq_32k_h32"):
            rr = measure(WORKLOADS[name], 5, 3, dev, rank, dist)
            extra[name] = {"ms_per_step": rr["total_ms"] / 5,
                           "Mtokens_s": job_mtokens_s(rr["alg"]["tokens"], world, 5, rr["total_ms"]),
                           "fwd": rr["fwd"], "bwd": rr["bwd"], "fwd_infer": rr["fwd_infer"],
                           "kernels_us": {k: 1e3 * v[1] / v[0] for k, v in rr["rep"].items()}}
            del rr

    # every rank takes this collective, so a device error on one rank ends all of them
    # here rather than leaving the others waiting at the next barrier
    status = int(max_over_ranks(gdn.device_status(), dist, dev))
    if status != 0:
        if dist:
            dist.destroy_process_group()
        raise SystemExit(f"device status {status} after the bench (max over ranks)")

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args, w)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "Mtokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "T": w.T, "Hq": w.Hq, "Hv": w.Hv, "K": w.K,
                       "V": w.V, "chunk": CHUNK, "step": "fwd+bwd" if do_bwd else "fwd",
                       "l2": "flushed between steps (2x L2 write, outside the events)",
                       "parallelism": f"replicas x{world} (independent sequences per GPU)"},
            "fwd": None, "bwd": None, "fwd_infer": None,
            "kernels": kernels, "roofline": roofline,
            "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": int(round(sum(v[0] for v in rep.values()))),
            "clocks": clk.summary(),
        }
        line["fwd"], line["bwd"], line["fwd_infer"] = fwd_blocks
        if extra:
            line["other_workloads"] = extra
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
