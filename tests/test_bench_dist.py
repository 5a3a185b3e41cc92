"""bench.py's multi-rank plumbing on CPU: two gloo ranks (no GPU needed).

Covers what the N > 1 launch adds around the single-GPU step: the process
group, the MAX reduction of per-rank times, the barrier, per-rank workloads,
and the reference arm printing exactly one line from rank 0 under torchrun.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    from dsa_workloads import CONFIGS, make_workload
    import torch.distributed as dist
    w, r, _ = bench.dist_setup(None, backend="gloo")
    try:
        local_ms = 1.0 + 2.0 * r                 # rank 1 is the slow one
        m = bench.reduce_max(local_ms, w)
        bench.barrier(w)
        spec = bench.rank_spec(CONFIGS["tiny_prefill_1k"], r)
        wl = make_workload(spec)
        q.put((r, w, m, spec.seed, float(wl.q[0, 0, :8].float().sum())))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_and_workloads():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=10) for _ in range(2))
    (r0, w0, m0, s0, v0), (r1, w1, m1, s1, v1) = got
    assert (r0, r1) == (0, 1) and w0 == w1 == 2
    assert m0 == m1 == 3.0                       # every rank sees the slowest rank's time
    assert s0 != s1 and v0 != v1                 # each rank serves its own batch


def test_reference_arm_under_torchrun_two_ranks():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0", "--config", "tiny_prefill_1k"]
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=600, env=env, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, res.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
    # the line carries every key of the bench contract
    keys = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
            "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"}
    assert keys <= set(d), keys - set(d)
    assert d["steps"] == 1 and d["warmup"] == 0 and d["higher_is_better"] is True
    assert d["config"]["workload"] == "tiny_prefill_1k"
    assert d["e2e"]["value"] == d["value"] and d["e2e"]["unit"] == d["unit"] == d["cpu_baseline"]["unit"]
    assert {"value", "cores", "sample"} <= set(d["cpu_baseline"]) and d["cpu_baseline"]["value"] == d["value"]
