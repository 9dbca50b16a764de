"""The multi-rank (N > 1) plumbing, on the CPU with the gloo backend.

bench.py runs one independent sequence per rank (batch sharding, no collective on the
data path) and reports the job time as the max over ranks.  These tests run that
plumbing in two processes: the max reduction, the per-rank seeding, and the reference
arm's launch contract under torchrun (rank 0 alone prints one JSON line).

The KV-group shard of one layer (token_sparse_attention_dtc_b200.shard) has one real
exchange: the all-gather of every rank's partial layer score.  Its test runs two ranks
on CPU tensors, each scoring its own heads with the oracle, and checks that the
exchange puts rank r's partial at index r identically on both ranks, and that the
budget on the rank-order combination is bit-exact against the oracle's budget on the
unsharded layer's scores.
"""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
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


def _shard_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import oracle
    from token_sparse_attention_dtc_b200 import shard
    from token_sparse_attention_dtc_b200.inputs import make_inputs

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, L, H, Hkv, d, qn = 2, 600, 8, 4, 64, 16
        x = make_inputs(B, L, H, Hkv, d, torch.bfloat16, seed=5)   # the same on every rank
        h0, h1 = shard.head_range(H, Hkv, rank, world)
        kv0, kv1 = shard.kv_group_range(Hkv, rank, world)
        Qr = x["Q"][:, :, h0:h1].contiguous()
        Kr = x["K"][:, :, kv0:kv1].contiguous()
        s_h, _ = oracle.score(Qr, Kr, qn)                          # this rank's heads
        u = np.zeros((B, L))
        for h in range(h1 - h0):                                   # head order
            u += s_h[:, h]
        parts = shard.exchange_partials(torch.from_numpy(u.astype(np.float32)))
        q.put((rank, (h0, h1, kv0, kv1), parts.numpy()))
    finally:
        dist.destroy_process_group()


def test_kv_group_shard_exchange_and_budget_match_the_unsharded_layer():
    import oracle
    from token_sparse_attention_dtc_b200.inputs import make_inputs

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted([q.get(timeout=300) for _ in range(2)], key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert out[0][1] == (0, 4, 0, 2) and out[1][1] == (4, 8, 2, 4)
    parts0, parts1 = out[0][2], out[1][2]
    assert parts0.shape == (2, 2, 600) and np.array_equal(parts0, parts1)
    # the combination every rank performs: partials summed in rank order, normalised
    u = parts0[0].astype(np.float64) + parts0[1].astype(np.float64)
    s_l = (u / u.sum(axis=1, keepdims=True)).astype(np.float32)
    x = make_inputs(2, 600, 8, 4, 64, torch.bfloat16, seed=5)
    ref_h, ref_l = oracle.score(x["Q"], x["K"], 16)
    assert np.max(np.abs(s_l - ref_l) / ref_l) <= 1e-6
    for tau in (0.005, 0.02, 0.2):
        lk, _ = oracle.budget(s_l, tau)
        want, _ = oracle.budget(ref_l.astype(np.float32), tau)
        np.testing.assert_array_equal(lk, want)


@pytest.mark.parametrize("Hkv,world", [(8, 1), (8, 2), (8, 3), (8, 8), (4, 3), (1, 1)])
def test_kv_group_ranges_cover_every_group_once(Hkv, world):
    from token_sparse_attention_dtc_b200 import shard

    spans = [shard.kv_group_range(Hkv, r, world) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == Hkv
    assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
    sizes = [b - a for a, b in spans]
    assert min(sizes) >= 1 and max(sizes) - min(sizes) <= 1
    H = 4 * Hkv
    assert [shard.head_range(H, Hkv, r, world) for r in range(world)] == [
        (4 * a, 4 * b) for a, b in spans]


def test_kv_group_range_rejects_more_ranks_than_groups():
    from token_sparse_attention_dtc_b200 import shard

    with pytest.raises(ValueError):
        shard.kv_group_range(2, 0, 3)
