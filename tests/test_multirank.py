"""The multi-rank (N > 1) plumbing of bench.py, on the CPU with the gloo backend.

bench.py runs one independent sequence per rank (batch sharding, no collective on the
data path) and reports the job time as the max over ranks.  These tests run that
plumbing in two processes: the max reduction, the per-rank seeding, and the reference
arm's launch contract under torchrun (rank 0 alone prints one JSON line).
"""
import json
import os
import socket
import subprocess
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    from token_sparse_attention_dtc_b200.inputs import make_workload

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local = [12.5, 40.25][rank]
        job = bench.job_max(local, world, "cpu")
        x = make_workload("tiny_mha_1k", seed=bench.rank_seed(0, rank), L=64)
        q.put((rank, job, float(x["Q"].double().sum())))
    finally:
        dist.destroy_process_group()


def test_job_time_is_max_over_ranks_and_ranks_draw_distinct_inputs():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort()
    assert out[0][1] == out[1][1] == 40.25
    assert out[0][2] != out[1][2]


def test_reference_arm_under_torchrun_prints_one_line_on_rank_zero():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py",
           "--impl", "reference", "--gpus", "2", "--workload", "tiny_mha_1k", "--L", "256",
           "--steps", "1", "--warmup", "0"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["unit"] == "ms"
    assert d["higher_is_better"] is False and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0
