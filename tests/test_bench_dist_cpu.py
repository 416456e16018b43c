"""The multi-rank path of bench.py on CPU: two gloo ranks on 127.0.0.1.

With N GPUs every rank runs its own independent batch (no collective on the
data path); the job's time is the slowest rank's, taken by an all-reduce MAX,
and its throughput is all ranks' tokens over that time. These are the host-side
pieces of that path; the per-rank device work is the single-GPU path the GPU
tests cover."""
import json
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out_dir):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    from gated_deltanet_chunked_rule_b200.inputs import Workload, make_inputs
    ws, r, local = bench.dist_setup()
    dist.init_process_group("gloo", rank=r, world_size=ws)
    try:
        w = Workload("dist", B=1, T=96, Hq=1, Hv=2, K=64, V=64, seed=7)
        wr = bench.rank_workload(w, r)
        x = make_inputs(wr)
        # this rank's own (deliberately different) device time
        mine = 3.0 + 2.0 * r
        job = bench.slowest_ms(mine, dist, "cpu")
        # a device status seen on one rank only reaches every rank
        status = int(bench.max_over_ranks(6 if r == 1 else 0, dist, "cpu"))
        value = bench.job_mtokens_s(w.B * w.T, ws, 4, job)
        dist.barrier()
        with open(os.path.join(out_dir, f"rank{r}.json"), "w") as f:
            json.dump({"rank": r, "local": local, "seed": wr.seed, "q_sum": float(x["q"].double().sum()),
                       "job_ms": job, "value": value, "status": status}, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_time_max_and_independent_batches(tmp_path):
    world = 2
    mp.start_processes(_rank, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn",
                       join=True)
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    assert [x["rank"] for x in res] == [0, 1] and [x["local"] for x in res] == [0, 1]
    # every rank sees the slowest rank's time
    assert res[0]["job_ms"] == res[1]["job_ms"] == pytest.approx(5.0)
    # whole-job throughput: both ranks' tokens over that time
    assert res[0]["value"] == pytest.approx(96 * 2 * 4 / 5.0e-3 / 1e6)
    assert res[0]["status"] == res[1]["status"] == 6
    # independent batches: different seeds, different inputs
    assert res[0]["seed"] != res[1]["seed"] and res[0]["q_sum"] != res[1]["q_sum"]


def test_single_rank_needs_no_collective():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.slowest_ms(4.25) == 4.25
    assert bench.job_mtokens_s(8192, 1, 10, 8.0) == pytest.approx(8192 * 10 / 8e-3 / 1e6)


def test_gpus_flag_launches_that_many_ranks():
    """`bench.py --gpus 2` outside torchrun relaunches itself with two local ranks
    (torch.distributed.run on 127.0.0.1); the host-side self-test of that path runs
    on gloo, so the line's n_gpus and max-over-ranks time come from two processes."""
    import subprocess
    import sys
    env = dict(os.environ)
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT"):
        env.pop(k, None)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--dist-selftest"],
                       capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    assert lines[0]["n_gpus"] == 2 and lines[0]["selftest"]
    # rank r reports 1 + r ms: the job's time is the slower rank's
    assert lines[0]["ms_per_step"] == pytest.approx(2.0)
