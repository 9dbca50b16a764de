"""Benchmark of the Token Sparse Attention layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload llama8b_128k] [--no-dense] [--no-e2e] [--no-cpu-baseline]

A step is one sparse layer (score, budget, select, gather, attention, scatter +
residual) on one sequence of the workload, inputs resident in HBM.  Prints one JSON
line on rank 0.  With N > 1 (torchrun) every rank runs its own sequence (batch
sharded, no collective on the data path): weak scaling, time = max over ranks.

--impl reference times the CPU oracle (the fp64 restatement of the pages' method) on
the host cores, each step a bounded sample of the same workload.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "token-sparse attn layer ms @128K Llama-8B shape; TFLOP/s & % roofline"
STAGES = ("score", "budget", "select", "gather", "attn", "scatter")
# fractions of the tokens pruned at 128K in the pages' own runs (L' = 0.456 L and 0.326 L)
PAGES_SPARSITY = (0.544, 0.674)
# thresholds of the block-sparse pattern (blocks within theta of a pair's best block mean)
BLOCK_THETAS = (0.25, 0.1)


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"],
                    bf16_sus=d.get("bf16_tflops_sustained", d["bf16_tflops"]), src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


def _traffic_key(w, L: int):
    """The traffic.json key of a workload run at length L: its name at its own length, none
    when --L changed the size (a capture of another length does not apply)."""
    return w.name if L == w.L else None


def _traffic(kernel: str, workload):
    """DRAM bytes per launch from the committed ncu summary, if it still matches the source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel, {}).get(workload) if workload else None
    if not e:
        return None
    import hashlib

    src = os.path.join(ROOT, "token_sparse_attention_dtc_b200", "csrc", e["source"])
    if not os.path.exists(src):
        return None
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    return e["bytes_per_launch"] if h == e["source_sha"] else None


def score_kernel_name(schedule: str, w, L: int, B: int = 1, sms: int = 148) -> str:
    """The bf16 scoring kernel the library runs for this schedule and shape (the rule of
    tsa_set_score_schedule in include/tsa.h): the wave-scheduled kernel covers q_eff = 16,
    at most 4 query heads per KV head and d = 64 or 128; the automatic schedule takes it
    (every KV group in one wave) when K holds at least 192 MiB and B * Hkv fits the SMs."""
    covered = (str(w.dtype) == "torch.bfloat16" and min(w.q, L) == 16 and w.H // w.Hkv <= 4
               and w.d in (64, 128) and L >= 16)
    kbytes = 2.0 * B * L * w.Hkv * w.d
    if covered and (schedule == "wave" or
                    (schedule == "auto" and kbytes >= 192.0 * (1 << 20)
                     and B * w.Hkv <= min(sms, 160))):
        return "k_score_wave"
    return "k_score_tc" if str(w.dtype) == "torch.bfloat16" else "k_score_simt"


def l2_note(d) -> str:
    """Whether the timed inputs exceed the 126 MB L2 (no flush is done between steps)."""
    mb = {k: d[k].numel() * d[k].element_size() / 1e6 for k in ("Q", "K", "V", "X")}
    big = all(v > 126 for v in mb.values())
    return ("inputs larger than L2 (Q %.0f MB, K/V %.0f MB each, X %.0f MB); no flush"
            % (mb["Q"], mb["K"], mb["X"]) if big else
            "inputs not all larger than L2 (Q %.0f MB, K/V %.0f MB each, X %.0f MB); no flush"
            % (mb["Q"], mb["K"], mb["X"]))


def block_useful_flops(mask, lk: int, d: int) -> float:
    """Useful attention FLOPs (QK^T and PV, causal keys of kept blocks) of a block mask
    [B=1, H, NP, NW] int32 for L' = lk: 4 d per visible (query, key) pair."""
    import numpy as np
    m = mask.cpu().numpy().view(np.uint32)[0]          # [H, NP, NW]
    H, NP, NW = m.shape
    bits = ((m[..., :, None] >> np.arange(32, dtype=np.uint32)) & 1).reshape(H, NP, NW * 32)
    total = 0.0
    for p in range((lk + 255) // 256):
        kept = bits[:, p, :]                           # [H, NB]
        for x in (0, 1):
            r0 = 256 * p + 128 * x
            rows = max(0, min(128, lk - r0))
            if rows == 0:
                continue
            full = kept[:, : 2 * p + x].sum(axis=1) * 128.0       # blocks before the diagonal
            diag = rows * (rows + 1) / 2.0                        # the tile's own block
            total += float((full * rows + diag * kept[:, 2 * p + x]).sum())
    return 4.0 * d * total


def kv_union_rows(idx, lk: int, Hkv: int) -> int:
    """Rows of K (and of V) a gather must read: per KV head, the tokens kept by at least
    one of its query heads (idx is [B, H, L], its first lk entries per row kept)."""
    import torch
    B, H, L = idx.shape
    kept = idx[:, :, :lk].reshape(B, Hkv, (H // Hkv) * lk).long()
    mask = torch.zeros(B, Hkv, L, dtype=torch.bool, device=idx.device)
    mask.scatter_(2, kept, True)
    return int(mask.sum().item())


def rank_seed(seed: int, rank: int) -> int:
    """Each rank draws its own sequence (batch sharding)."""
    return seed * 1000 + rank


def job_max(value: float, world: int, device=None) -> float:
    """Max of a per-rank value over all ranks (the job's time); identity on one rank."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist

    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.Q,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        rows = []
        for line in (self.out or "").strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 8:
                continue
            try:
                rows.append((float(f[0]), float(f[1]), f[4:8]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({names[i] for _, _, r in rows for i in range(4) if r[i] == "Active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": rows[0][1],
                "samples": len(rows), "reasons": reasons}


def _workload_desc(w, L):
    return ("%s: B=1 per GPU, L=%d, H=%d, Hkv=%d, d=%d, bf16, q=%d, tau=%g, 4 sinks + "
            "%.1f%% heavy hitters shifted %.1f along per-group query directions"
            % (w.name, L, w.H, w.Hkv, w.d, w.q, w.tau, 100 * w.heavy_frac, w.shift))


# --------------------------------------------------------------------------- oracle ---

def host_cpu():
    """Host cores the oracle may use and the CPU model (from /proc/cpuinfo)."""
    try:
        usable = len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        usable = os.cpu_count() or 1
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return dict(nproc=usable, cpu_count=os.cpu_count(), model=model)


def oracle_sample(x, w, L, attn_budget_s=30.0, slice_div=64):
    """Time the oracle on one layer: scoring, budget and selection in full; attention on
    whole heads when they fit in attn_budget_s (all of them at small L), else on a
    strided sample of head 0's rows, extrapolated by exact causal pair count;
    decompress + residual on 1/slice_div of the tokens, scaled by token count.  Returns
    (ms per full layer, sample description, info, seconds spent)."""
    import numpy as np

    import oracle

    cpu = host_cpu()
    threads = cpu["nproc"]
    t_spent = time.perf_counter()
    t0 = time.perf_counter()
    s_h, s_l = oracle.score(x["Q"], x["K"], w.q, nthreads=threads)
    t1 = time.perf_counter()
    lk, _ = oracle.budget(s_l.astype(np.float32), w.tau)
    t2 = time.perf_counter()
    idx = oracle.select(s_h.astype(np.float32), lk)
    t3 = time.perf_counter()
    Lk = int(lk[0])
    # attention: whole heads, one after another, while the next one is expected to fit in
    # attn_budget_s (every head costs the same: each keeps L' rows); if even one head is
    # not expected to fit (from a rate measured on 32 rows of head 0), every k-th row of
    # head 0 instead
    pairs_head = Lk * (Lk + 1) / 2.0
    pairs_full = w.H * pairs_head
    t_attn_meas, pairs_done, rows_timed, heads_done, stride = 0.0, 0.0, 0, 0, 0
    if Lk:
        cal = sorted(set(np.linspace(0, Lk - 1, 32).astype(int).tolist()))
        tc0 = time.perf_counter()
        oracle.attend_rows(x["Q"], x["K"], x["V"], idx, lk, [(0, 0, i) for i in cal],
                           nthreads=threads)
        rate = sum(i + 1 for i in cal) / max(time.perf_counter() - tc0, 1e-6)
        if pairs_head / rate <= attn_budget_s:
            per_head = pairs_head / rate
            while heads_done < w.H and t_attn_meas + per_head <= attn_budget_s:
                ta = time.perf_counter()
                oracle.attend_rows(x["Q"], x["K"], x["V"], idx, lk,
                                   [(0, heads_done, i) for i in range(Lk)], nthreads=threads)
                per_head = time.perf_counter() - ta
                t_attn_meas += per_head
                heads_done += 1
            pairs_done, rows_timed = heads_done * pairs_head, heads_done * Lk
        else:
            stride = max(2, int(math.ceil(pairs_head / max(attn_budget_s * rate, 1.0))))
            rows_i = list(range(stride // 2, Lk, stride))
            ta = time.perf_counter()
            oracle.attend_rows(x["Q"], x["K"], x["V"], idx, lk, [(0, 0, i) for i in rows_i],
                               nthreads=threads)
            t_attn_meas = time.perf_counter() - ta
            pairs_done, rows_timed = float(sum(i + 1 for i in rows_i)), len(rows_i)
    factor = pairs_full / pairs_done if pairs_done else 1.0
    t_attn = t_attn_meas * factor
    # decompress + residual: in full while its fp64 arrays stay small (up to 2^25
    # elements each), else on 1/slice_div of the tokens, scaled by token count
    n = L if L * w.H * w.d <= (1 << 25) else max(1, L // slice_div)
    Oh = np.zeros((1, w.H, n, w.d))
    idx_s = np.tile(np.arange(n, dtype=np.int32), (1, w.H, 1))
    td0 = time.perf_counter()
    oracle.decompress_residual(Oh, idx_s, np.array([min(Lk, n)], np.int32), x["X"][:, :n])
    td1 = time.perf_counter()
    t_dec = (td1 - td0) * L / n
    total = (t1 - t0) + (t2 - t1) + (t3 - t2) + t_attn + t_dec
    measured = (t1 - t0) + (t2 - t1) + (t3 - t2) + t_attn_meas + (td1 - td0)
    if Lk == 0 or factor == 1.0:
        attn_desc = "attention in full (%d heads x %d rows)" % (w.H, Lk)
    elif heads_done:
        attn_desc = ("attention on %d whole head(s) of %d (%d rows each), x%.4g by causal "
                     "pair count" % (heads_done, w.H, Lk, factor))
    else:
        attn_desc = ("attention on every %d-th row of head 0 (%d of %d rows), x%.4g to all "
                     "%d heads by causal pair count" % (stride, rows_timed, Lk, factor, w.H))
    info = dict(score_s=t1 - t0, budget_s=t2 - t1, select_s=t3 - t2,
                attn_s_measured=t_attn_meas, attn_extrapolation_factor=factor,
                attn_s_extrapolated=t_attn, attn_rows_timed=rows_timed,
                decompress_s_measured=td1 - td0, decompress_extrapolation_factor=L / n,
                Lkeep=Lk, threads=threads, nproc=cpu["nproc"], cpu_count=cpu["cpu_count"],
                cpu_model=cpu["model"], measured_s=measured,
                measured_fraction=measured / total if total > 0 else 1.0,
                wall_s=time.perf_counter() - t_spent)
    dec_desc = ("decompress+residual in full" if n == L else
                "decompress+residual on %d of %d tokens, x%d" % (n, L, L // n))
    sample = ("scoring, budget and selection in full on the %d-token sequence; %s; %s; "
              "%.3g%% of the layer's oracle time measured%s; %d threads on %s"
              % (L, attn_desc, dec_desc, 100.0 * info["measured_fraction"],
                 "" if info["measured_fraction"] >= 0.9999 else ", the rest extrapolated",
                 threads, cpu["model"]))
    return total * 1e3, sample, info, measured


def run_reference(args, w, L, rank, world):
    if rank != 0:
        return
    from token_sparse_attention_dtc_b200.inputs import make_workload

    x = make_workload(w.name, seed=args.seed, L=L, B=1)
    times = []
    sample = info = None
    for s in range(args.warmup + args.steps):
        # each step a bounded sample: a few seconds of attention on the host cores
        ms, sample, info, _ = oracle_sample(x, w, L, attn_budget_s=args.ref_attn_seconds)
        if s >= args.warmup:
            times.append(ms)
    v = statistics.mean(times)
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "ms", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": v,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": _workload_desc(w, L), "oracle": "fp64 C, pthreads"},
        "cpu_baseline": {"value": v, "unit": "ms", "cores": info["threads"], "kind": "oracle",
                         "sample": sample, "nproc": info["nproc"], "cpu_model": info["cpu_model"],
                         "measured_fraction": info["measured_fraction"],
                         "attn_extrapolation_factor": info["attn_extrapolation_factor"]},
        "e2e": {"value": v, "unit": "ms", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "oracle_breakdown_s": info,
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- ours ---

def run_ours(args, w, L, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from token_sparse_attention_dtc_b200 import tsa
    from token_sparse_attention_dtc_b200.inputs import make_workload

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    tsa.lib()  # fail loudly if the CUDA library is missing
    x = make_workload(w.name, seed=rank_seed(args.seed, rank), L=L, B=1)
    d = {k: v.to(dev) for k, v in x.items()}
    dm = tsa.dims(d["Q"], d["K"])
    ws = tsa.workspace(dm, w.q, layer=True, device=dev)
    Y = torch.empty_like(d["X"])
    Lk = torch.empty(1, dtype=torch.int32, device=dev)
    idx = torch.empty(1, w.H, L, dtype=torch.int32, device=dev)
    st = torch.cuda.current_stream(dev)

    def sync_all():
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()

    n_ev = 7
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
           for _ in range(args.steps)]
    for row in evs:
        for e in row:
            e.record(st)  # materialise the event handles
    for _ in range(args.warmup):
        tsa.tsa_layer(d["Q"], d["K"], d["V"], d["X"], Y, q=w.q, tau=w.tau, Lkeep=Lk, idx=idx,
                      ws=ws)
    sync_all()
    if tsa.tsa_get_device_status(ws) != 0:
        raise RuntimeError("device error during warm-up")
    t_start = torch.cuda.Event(enable_timing=True)
    t_stop = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        time.sleep(0.3)
        sync_all()
        n_launch0 = tsa.kernel_launches()
        t_start.record(st)
        for s in range(args.steps):
            tsa.tsa_layer(d["Q"], d["K"], d["V"], d["X"], Y, q=w.q, tau=w.tau, Lkeep=Lk,
                          idx=idx, ws=ws)
        t_stop.record(st)
        n_launches = tsa.kernel_launches() - n_launch0
        sync_all()
    total_ms = t_start.elapsed_time(t_stop)
    ms_step = total_ms / args.steps
    # The stage breakdown: the same steps again, with an event between every two stages
    # (the events hold each kernel back until the one before it has finished, so this
    # loop's layer time is reported on its own).
    sync_all()
    t_start.record(st)
    for s in range(args.steps):
        tsa.tsa_layer(d["Q"], d["K"], d["V"], d["X"], Y, q=w.q, tau=w.tau, Lkeep=Lk,
                      idx=idx, ws=ws, stage_events=evs[s])
    t_stop.record(st)
    sync_all()
    ms_step_staged = job_max(t_start.elapsed_time(t_stop) / args.steps, world, dev)
    stage_ms = {name: statistics.mean(evs[s][i].elapsed_time(evs[s][i + 1])
                                      for s in range(args.steps))
                for i, name in enumerate(STAGES)}
    lk = int(Lk.item())
    if tsa.tsa_get_device_status(ws) != 0:
        raise RuntimeError("device error during the timed region")
    ms_step = job_max(ms_step, world, dev)

    peaks = _peaks()
    flops = 2.0 * w.H * w.d * lk * (lk + 1)
    attn_ms = stage_ms["attn"]
    attn_tf = flops / (attn_ms * 1e-3) / 1e12
    roof = {"kernel": "k_attn_tc", "bound": "tensor", "achieved": attn_tf,
            "peak": peaks["bf16_sus"], "unit": "TFLOP/s", "frac": attn_tf / peaks["bf16_sus"],
            "peak_kind": "bf16 sustained (%s)" % peaks["src"],
            "frac_of_burst": attn_tf / peaks["bf16"],
            "traffic": _traffic("k_attn_tc", _traffic_key(w, L))}
    # HBM kernels: algorithmic bytes per launch
    H, dd = w.H, w.d
    hbm = {
        "score": (L * w.Hkv * dd * 2 + w.q * H * dd * 2 + 4 * H * L + 4 * L),
        # Q rows read and Qh, Kh, Vh written once per query head; K and V rows read once
        # per KV head over the union of its query heads' kept sets (the shared rows are
        # L2 hits)
        "gather": 4 * H * lk * dd * 2 + 2 * kv_union_rows(idx, lk, w.Hkv) * dd * 2,
        "scatter": 2 * L * H * dd * 2 + H * lk * dd * 2 + 4 * H * L,
    }
    hbm_roof = {k: {"ms": stage_ms[k], "achieved_gbs": v / (stage_ms[k] * 1e-3) / 1e9,
                    "frac": v / (stage_ms[k] * 1e-3) / 1e9 / peaks["hbm"],
                    "algorithmic_bytes": v}
                for k, v in hbm.items()}
    # ncu-counted DRAM bytes of the committed capture, when it matches the source
    score_kern = score_kernel_name(args.score_schedule, w, L)
    for k, kern in (("score", score_kern), ("gather", "k_gather_qkv"),
                    ("scatter", "k_scatter_residual")):
        t = _traffic(kern, _traffic_key(w, L))
        hbm_roof[k]["traffic"] = t
        hbm_roof[k]["dram_gbs"] = t / (stage_ms[k] * 1e-3) / 1e9 if t else None
        hbm_roof[k]["dram_frac"] = (t / (stage_ms[k] * 1e-3) / 1e9 / peaks["hbm"]) if t else None

    # the scoring kernel on its own: the layer loop's score stage also absorbs the
    # write-back of the previous scatter's dirty Y lines from L2 and the launch gap, so
    # time the kernel after a flush that leaves L2 clean (a read of 512 MB after a write),
    # with enough work queued ahead that the GPU never waits for the host
    score_iso = None
    if w.dtype == torch.bfloat16:
        flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
        s_h_i = torch.empty(1, w.H, L, device=dev)
        s_l_i = torch.empty(1, L, device=dev)
        ws_i = tsa.workspace(dm, w.q, device=dev)
        for _ in range(3):
            tsa.tsa_score(d["Q"], d["K"], w.q, s_h=s_h_i, s_l=s_l_i, ws=ws_i)
        sync_all()
        iso = []
        for _ in range(max(5, args.steps)):
            flush.zero_()
            flush.view(torch.int32).max()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(st)
            tsa.tsa_score(d["Q"], d["K"], w.q, s_h=s_h_i, s_l=s_l_i, ws=ws_i)
            b.record(st)
            b.synchronize()
            iso.append(a.elapsed_time(b))
        if tsa.tsa_get_device_status(ws_i) != 0:
            raise RuntimeError("device error in the isolated scoring runs")
        score_iso = statistics.median(iso)
        del flush, s_h_i, s_l_i, ws_i

    if score_iso is not None:
        v = hbm["score"]
        hbm_roof["score"]["kernel_ms_isolated"] = score_iso
        hbm_roof["score"]["isolated_achieved_gbs"] = v / (score_iso * 1e-3) / 1e9
        hbm_roof["score"]["isolated_frac"] = v / (score_iso * 1e-3) / 1e9 / peaks["hbm"]
        t = hbm_roof["score"].get("traffic")
        if t:
            hbm_roof["score"]["isolated_dram_frac"] = t / (score_iso * 1e-3) / 1e9 / peaks["hbm"]

    # dense causal attention through the same kernel, same shape
    dense = None
    if not args.no_dense:
        for _ in range(2):
            tsa.tsa_layer(d["Q"], d["K"], d["V"], d["X"], Y, is_sparse=False, ws=ws)
        # As many layers as the sparse loops, timed the same way: the layer without stage
        # events, then the attention from a second loop with them.
        nd = args.steps
        dev_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(7)] for _ in range(nd)]
        for row in dev_ev:
            for e in row:
                e.record(st)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        sync_all()
        a.record(st)
        for _ in range(nd):
            tsa.tsa_layer(d["Q"], d["K"], d["V"], d["X"], Y, is_sparse=False, ws=ws)
        b.record(st)
        sync_all()
        dms = job_max(a.elapsed_time(b) / nd, world, dev)
        for i in range(nd):
            tsa.tsa_layer(d["Q"], d["K"], d["V"], d["X"], Y, is_sparse=False, ws=ws,
                          stage_events=dev_ev[i])
        sync_all()
        dflops = 2.0 * w.H * w.d * L * (L + 1)
        dattn = statistics.mean(dev_ev[i][4].elapsed_time(dev_ev[i][5]) for i in range(nd))
        dense = {"layer_ms": dms, "attn_ms": dattn,
                 "attn_tflops": dflops / (dattn * 1e-3) / 1e12,
                 "attn_frac_of_sustained": dflops / (dattn * 1e-3) / 1e12 / peaks["bf16_sus"],
                 "speedup_sparse_vs_dense_layer": dms / ms_step}

    # the same layer captured once in a CUDA graph and replayed (no host launch gaps)
    graph = None
    try:
        side = torch.cuda.Stream(dev)
        side.wait_stream(st)
        with torch.cuda.stream(side):
            tsa.tsa_layer(d["Q"], d["K"], d["V"], d["X"], Y, q=w.q, tau=w.tau, Lkeep=Lk,
                          idx=idx, ws=ws)
        st.wait_stream(side)
        torch.cuda.synchronize(dev)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            tsa.tsa_layer(d["Q"], d["K"], d["V"], d["X"], Y, q=w.q, tau=w.tau, Lkeep=Lk,
                          idx=idx, ws=ws)
        g.replay()
        sync_all()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(st)
        for _ in range(args.steps):
            g.replay()
        b.record(st)
        sync_all()
        graph = {"layer_ms": job_max(a.elapsed_time(b) / args.steps, world, dev) / world}
        del g
    except Exception as e:  # reported, not required
        graph = {"error": str(e).splitlines()[0][:200]}

    # the whole layer at the pages' sparsities (54.4% and 67.4% of the tokens pruned at
    # 128K), through the fixed-ratio budget on the same synthetic inputs
    pages = None
    if not args.no_pages_sparsity:
        pages = []
        for sp in PAGES_SPARSITY:
            lk_p = L - int(math.floor(sp * L))
            for _ in range(2):
                tsa.tsa_layer(d["Q"], d["K"], d["V"], d["X"], Y, q=w.q, ws=ws, sparsity=sp)
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(7)]
            for e in ev:
                e.record(st)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            sync_all()
            a.record(st)
            npg = 2
            for _ in range(npg):
                tsa.tsa_layer(d["Q"], d["K"], d["V"], d["X"], Y, q=w.q, ws=ws, sparsity=sp,
                              stage_events=ev)
            b.record(st)
            sync_all()
            pms = job_max(a.elapsed_time(b) / npg, world, dev)
            pattn = ev[4].elapsed_time(ev[5])
            pfl = 2.0 * w.H * w.d * lk_p * (lk_p + 1)
            pages.append({"pruned": sp, "Lkeep": lk_p, "layer_ms": pms, "attn_ms": pattn,
                          "attn_tflops": pfl / (pattn * 1e-3) / 1e12,
                          "speedup_vs_dense_layer": (dense["layer_ms"] / pms) if dense else None,
                          "data": "pages' sparsity, synthetic (fixed-ratio budget)"})
        if tsa.tsa_get_device_status(ws) != 0:
            raise RuntimeError("device error in the pages'-sparsity runs")

    # the fused compress + attention + decompress (direct gather) against the staged layer,
    # at the synthetic budget and, for long sequences, at the pages' 67.4% pruned
    direct = None
    if not args.no_pages_sparsity and w.dtype == torch.bfloat16:
        direct = []
        cases = [("synthetic budget", dict(tau=w.tau))]
        if L >= 65536:
            cases.append(("67.4% pruned", dict(sparsity=PAGES_SPARSITY[1])))
        for name, kw in cases:
            row = {"case": name}
            for mode in (False, True):
                for _ in range(2):
                    tsa.tsa_layer(d["Q"], d["K"], d["V"], d["X"], Y, q=w.q, ws=ws, direct=mode, **kw)
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                sync_all()
                nrep = 3 if L >= 65536 else 20
                a.record(st)
                for _ in range(nrep):
                    tsa.tsa_layer(d["Q"], d["K"], d["V"], d["X"], Y, q=w.q, ws=ws, direct=mode,
                                  **kw)
                b.record(st)
                sync_all()
                row["direct_ms" if mode else "staged_ms"] = job_max(a.elapsed_time(b) / nrep,
                                                                    world, dev)
            direct.append(row)
        if tsa.tsa_get_device_status(ws) != 0:
            raise RuntimeError("device error in the direct-gather runs")

    # token + block composition: block-sparse attention inside the compressed space
    blocks = None
    if not args.no_pages_sparsity and w.dtype == torch.bfloat16:  # tcgen05 path only
        blocks = []
        for th in BLOCK_THETAS:
            for _ in range(2):
                tsa.tsa_layer(d["Q"], d["K"], d["V"], d["X"], Y, q=w.q, tau=w.tau, ws=ws,
                              block_theta=th)
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(7)]
            for e in ev:
                e.record(st)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            sync_all()
            a.record(st)
            for _ in range(2):
                tsa.tsa_layer(d["Q"], d["K"], d["V"], d["X"], Y, q=w.q, tau=w.tau, ws=ws,
                              block_theta=th, Lkeep=Lk, idx=idx, stage_events=ev)
            b.record(st)
            sync_all()
            bms = job_max(a.elapsed_time(b) / 2, world, dev)
            battn = ev[4].elapsed_time(ev[5])
            Qh, Kh, _ = tsa.tsa_gather_qkv(d["Q"], d["K"], d["V"], idx, Lk)
            _, bmask = tsa.tsa_block_select(dm, Qh, Kh, Lk, th, logits=False)
            del Qh, Kh
            lkb = int(Lk.item())
            useful = block_useful_flops(bmask, lkb, w.d)
            blocks.append({"theta": th, "Lkeep": lkb, "layer_ms": bms,
                           "attn_ms_incl_block_select": battn,
                           "useful_fraction_of_compressed": useful / (2.0 * w.H * w.d * lkb * (lkb + 1)),
                           "useful_attn_tflops": useful / (battn * 1e-3) / 1e12,
                           "speedup_vs_dense_layer": (dense["layer_ms"] / bms) if dense else None})
        torch.cuda.empty_cache()
        if tsa.tsa_get_device_status(ws) != 0:
            raise RuntimeError("device error in the block-sparse runs")

    # end to end through the public API with host buffers: every step copies its inputs
    # in from pinned host memory and its result out, inside the timed region.  Two device
    # slots let step k+1's inputs cross PCIe while step k computes (copy engines and SMs
    # in parallel): host-to-device stream, compute stream, device-to-host stream.
    e2e = None
    if not args.no_e2e:
        hx = {k: v.pin_memory() for k, v in x.items()}
        hY = [torch.empty(x["X"].shape, dtype=x["X"].dtype).pin_memory() for _ in range(2)]
        h2d = sum(v.numel() * v.element_size() for v in hx.values())
        d2h = hY[0].numel() * hY[0].element_size()
        slots = [d, {k: torch.empty_like(v) for k, v in d.items()}]
        Ys = [Y, torch.empty_like(Y)]
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev = lambda: torch.cuda.Event()
        in_ready, computed, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
        for e in computed + out_done:
            e.record(st)

        def e2e_step(k):
            s = k % 2
            with torch.cuda.stream(s_in):           # inputs of step k
                s_in.wait_event(computed[s])        # step k-2 no longer reads this slot
                for name in slots[s]:
                    slots[s][name].copy_(hx[name], non_blocking=True)
                in_ready[s].record(s_in)
            st.wait_event(in_ready[s])
            st.wait_event(out_done[s])              # step k-2's result has left this Y slot
            c = slots[s]
            tsa.tsa_layer(c["Q"], c["K"], c["V"], c["X"], Ys[s], q=w.q, tau=w.tau, ws=ws,
                          stream=st)
            computed[s].record(st)
            with torch.cuda.stream(s_out):          # result of step k
                s_out.wait_event(computed[s])
                hY[s].copy_(Ys[s], non_blocking=True)
                out_done[s].record(s_out)

        for k in range(2):
            e2e_step(k)
        sync_all()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        ne = max(4, args.steps)
        sync_all()
        a.record(s_in)
        for k in range(ne):
            e2e_step(k)
        s_out.wait_stream(st)
        b.record(s_out)
        sync_all()
        ems = job_max(a.elapsed_time(b) / ne, world, dev)
        e2e = {"value": ems / world, "unit": "ms", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "steps": ne,
               "overlap": "inputs of step k+1 copied in while step k computes"}
        del slots[1], Ys[1]

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        ms, sample, info, _ = oracle_sample(x, w, L, attn_budget_s=args.cpu_attn_seconds)
        cpu = {"value": ms, "unit": "ms", "cores": info["threads"], "kind": "oracle",
               "sample": sample, "nproc": info["nproc"], "cpu_model": info["cpu_model"],
               "measured_fraction": info["measured_fraction"],
               "attn_extrapolation_factor": info["attn_extrapolation_factor"],
               "breakdown_s": info}

    if rank == 0:
        line = {
            "metric": METRIC, "value": ms_step / world, "unit": "ms", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": _workload_desc(w, L), "global_batch": world, "seq_len": L,
                       "parallelism": "replicas (dp%d, no data-path collective)" % world,
                       "l2": l2_note(d), "score_schedule": args.score_schedule,
                       "score_kernel": score_kern,
                       "Lkeep": lk, "kept_fraction": lk / L},
            "roofline": roof,
            "stages_ms": stage_ms,
            "layer_ms_with_stage_events": ms_step_staged,
            "hbm_kernels": hbm_roof,
            "attn_tflops": attn_tf,
            "layer_tflops": flops / (ms_step * 1e-3) / 1e12,
            "overhead_fraction": 1.0 - attn_ms / sum(stage_ms.values()),
            "dense": dense,
            "graph_replay": graph,
            "pages_sparsity": pages,
            "block_sparse": blocks,
            "direct_gather": direct,
            "e2e": e2e,
            "cpu_baseline": cpu,
            "clocks": clk.summary(),
            "gpu_launches": n_launches,
            "peaks": peaks,
        }
        print(json.dumps(line), flush=True)


def run_stack(args, L):
    """32-layer stack (sparse and dense layers interleaved), one GPU.

    Fresh synthetic Q/K/V per layer (seed*1000 + layer), the residual stream X updated in
    place layer after layer.  The sparse set comes from the drift pass: an all-dense
    calibration run records X_0..X_32, tsa_drift ranks the layers, delta = 0.5 makes half
    of them sparse.  The stack is timed eagerly (one tsa_layer call per layer) and as a
    captured CUDA graph replay, against the all-dense stack."""
    import torch

    from token_sparse_attention_dtc_b200 import tsa
    from token_sparse_attention_dtc_b200.inputs import make_inputs

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    n_layers, H, Hkv, dd, q, tau = 32, 32, 8, 128, 16, 0.005
    layers = []
    for l in range(n_layers):
        x = make_inputs(1, L, H, Hkv, dd, torch.bfloat16, seed=args.seed * 1000 + l)
        layers.append({k: x[k].to(dev) for k in ("Q", "K", "V")})
    X0 = make_inputs(1, L, H, Hkv, dd, torch.bfloat16, seed=args.seed * 1000 + 999)["X"].to(dev)
    dm = tsa.dims(layers[0]["Q"], layers[0]["K"])
    ws = tsa.workspace(dm, q, layer=True, device=dev)
    X = X0.clone()
    st = torch.cuda.current_stream(dev)
    # L' of each sparse layer: rows of 4 int32, since optional outputs are 16-byte aligned
    Lk = torch.zeros(n_layers, 4, dtype=torch.int32, device=dev)

    def stack(mask):
        X.copy_(X0)
        for l in range(n_layers):
            c = layers[l]
            tsa.tsa_layer(c["Q"], c["K"], c["V"], X, X, is_sparse=bool(mask[l]), q=q, tau=tau,
                          Lkeep=Lk[l, :1], ws=ws)

    # calibration: all dense, keep every state for the drift pass
    states = torch.empty(n_layers + 1, L, H * dd, dtype=torch.bfloat16, device=dev)
    X.copy_(X0)
    states[0].copy_(X0[0])
    for l in range(n_layers):
        c = layers[l]
        tsa.tsa_layer(c["Q"], c["K"], c["V"], X, X, is_sparse=False, ws=ws)
        states[l + 1].copy_(X[0])
    R, mask_t = tsa.tsa_drift(states, eps=1e-6, delta=0.5)
    mask = [int(v) for v in mask_t.cpu()]
    del states

    def timed(fn, n=3):
        fn()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(st)
        for _ in range(n):
            fn()
        b.record(st)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / n

    n0 = tsa.kernel_launches()
    stack(mask)
    launches = tsa.kernel_launches() - n0
    eager_ms = timed(lambda: stack(mask))
    dense_ms = timed(lambda: stack([0] * n_layers))
    graph = {"replay_ms": None, "error": None}
    try:
        side = torch.cuda.Stream(dev)
        side.wait_stream(st)
        with torch.cuda.stream(side):
            stack(mask)          # warm the launchers outside capture
        st.wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            stack(mask)
        graph["replay_ms"] = timed(g.replay)
        Yg = X.clone()
        stack(mask)
        torch.cuda.synchronize()
        graph["replay_equals_eager"] = bool(torch.equal(Yg, X))
        del g
    except Exception as e:  # capture is reported, not required
        graph["error"] = str(e).splitlines()[0][:200]
    if tsa.tsa_get_device_status(ws) != 0:
        raise RuntimeError("device error in the stack run")
    line = {
        "metric": "32-layer stack ms (sparse set by drift, delta 0.5), Llama-8B heads",
        "value": graph["replay_ms"] or eager_ms, "unit": "ms", "n_gpus": 1,
        "higher_is_better": False, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "stack32: B=1, L=%d, H=32, Hkv=8, d=128, bf16, q=16, "
                               "tau=0.005, fresh Q/K/V per layer, X chained in place" % L},
        "eager_ms": eager_ms, "graph": graph, "all_dense_ms": dense_ms,
        "speedup_vs_all_dense": dense_ms / (graph["replay_ms"] or eager_ms),
        "sparse_layers": [l for l in range(n_layers) if mask[l]],
        "sparse_kept": [int(Lk[l, 0]) for l in range(n_layers) if mask[l]],
        "drift_R": [round(float(v), 6) for v in R.cpu()],
        "gpu_launches_per_stack": launches,
    }
    print(json.dumps(line), flush=True)


def run_sweep(args):
    """tau x q sweep on two 64K-token sequences (B = 2): one JSON line per setting."""
    import torch

    from token_sparse_attention_dtc_b200 import tsa
    from token_sparse_attention_dtc_b200.inputs import WORKLOADS, make_workload

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    name = "llama8b_64k_b2"
    x = make_workload(name, seed=args.seed)
    d = {k: v.to(dev) for k, v in x.items()}
    dm = tsa.dims(d["Q"], d["K"])
    Y = torch.empty_like(d["X"])
    Lk = torch.empty(dm.B, dtype=torch.int32, device=dev)
    st = torch.cuda.current_stream(dev)
    for q in (16, 64):
        ws = tsa.workspace(dm, q, layer=True, device=dev)
        for tau in (0.002, 0.005, 0.01, 0.02):
            run = lambda: tsa.tsa_layer(d["Q"], d["K"], d["V"], d["X"], Y, q=q, tau=tau,
                                        Lkeep=Lk, ws=ws)
            for _ in range(2):
                run()
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
            torch.cuda.synchronize()
            ev[0].record(st)
            for _ in range(3):
                run()
            ev[1].record(st)
            torch.cuda.synchronize()
            if tsa.tsa_get_device_status(ws) != 0:
                raise RuntimeError("device error in the sweep")
            ms = ev[0].elapsed_time(ev[1]) / 3
            lks = [int(v) for v in Lk.cpu()]
            fl = sum(2.0 * dm.H * dm.d * k * (k + 1) for k in lks)
            print(json.dumps({
                "metric": "token-sparse attn layer ms, tau x q sweep", "value": ms, "unit": "ms",
                "higher_is_better": False, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": _workload_desc(WORKLOADS[name], dm.L), "tau": tau,
                           "q": q, "B": dm.B},
                "Lkeep": lks, "kept_fraction": [k / dm.L for k in lks],
                "layer_tflops": fl / (ms * 1e-3) / 1e12}), flush=True)
        del ws


def run_drift(args):
    """Drift pass (tsa_drift) on Llama-8B-shaped calibration states: 32 layers + 1 states of
    T tokens x 4096, bf16 and fp32; one JSON line per shape with the HBM roofline.

    Algorithmic bytes: every state read once, (N + 1) * T * d_model * esize; the states are
    larger than L2 (no flush needed)."""
    import torch

    from token_sparse_attention_dtc_b200 import tsa

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    pk = _peaks()
    st = torch.cuda.current_stream(dev)
    for (N, T, D, dt) in ((32, 4096, 4096, torch.bfloat16), (32, 8192, 4096, torch.bfloat16),
                          (32, 4096, 4096, torch.float32)):
        g = torch.Generator(device="cpu").manual_seed(args.seed)
        h = torch.randn(N + 1, T, D, generator=g).to(dt).to(dev)
        ws = torch.zeros(tsa.lib().tsa_drift_workspace_size(N, T), dtype=torch.uint8, device=dev)
        for _ in range(max(args.warmup, 3)):
            tsa.tsa_drift(h, ws=ws)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        torch.cuda.synchronize()
        ev[0].record(st)
        for _ in range(args.steps):
            tsa.tsa_drift(h, ws=ws)
        ev[1].record(st)
        torch.cuda.synchronize()
        ms = ev[0].elapsed_time(ev[1]) / args.steps
        nbytes = h.numel() * h.element_size()
        gbs = nbytes / (ms * 1e-3) / 1e9
        # DRAM bytes of one launch, captured at 32 x 4096 x 4096 bf16; the bf16 walk reads
        # every row once, so the 8192-token launch is scaled by its token count.
        traffic = None
        t0 = _traffic("k_drift_walk", "drift_32x4096x4096_bf16")
        if t0 is not None and dt == torch.bfloat16 and (N, D) == (32, 4096):
            traffic = int(t0 * T / 4096)
        print(json.dumps({
            "metric": "drift pass ms (tsa_drift: R over N layers and the delta = 0.5 mask)",
            "value": ms, "unit": "ms", "higher_is_better": False,
            "dtype": "bf16" if dt == torch.bfloat16 else "f32", "data": "synthetic",
            "config": {"workload": "drift: N=%d layers, T=%d tokens, d_model=%d" % (N, T, D),
                       "l2": "states %.0f MB, larger than L2; no flush" % (nbytes / 1e6)},
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm"], "unit": "GB/s",
                         "frac": gbs / pk["hbm"], "traffic": traffic,
                         "algorithmic_bytes": nbytes}}), flush=True)
        del h, ws


def run_kv_shard(args, w, L, rank, world, local_rank):
    """One layer sharded by KV group over the job's ranks (token_sparse_attention_dtc_b200
    .shard): every rank draws the same layer, keeps its KV groups' heads, and runs its part
    (scoring of its heads, one NCCL all-gather of the partial layer scores, the rank-order
    combination, budget, selection, gather, attention, scatter).  A step is one layer of
    the whole job: strong scaling; the time is the max over ranks."""
    import torch
    import torch.distributed as dist

    from token_sparse_attention_dtc_b200 import shard, tsa
    from token_sparse_attention_dtc_b200.inputs import make_workload

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    tsa.lib()
    group = None
    if world == 1 and not dist.is_initialized():
        import datetime

        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        os.environ.setdefault("MASTER_PORT", "29512")
        dist.init_process_group("nccl", rank=0, world_size=1,
                                timeout=datetime.timedelta(seconds=300))
    x = make_workload(w.name, seed=args.seed, L=L, B=1)   # the same layer on every rank
    h0, h1 = shard.head_range(w.H, w.Hkv, rank, world)
    kv0, kv1 = shard.kv_group_range(w.Hkv, rank, world)
    d = {"Q": x["Q"][:, :, h0:h1].contiguous().to(dev),
         "K": x["K"][:, :, kv0:kv1].contiguous().to(dev),
         "V": x["V"][:, :, kv0:kv1].contiguous().to(dev),
         "X": x["X"][:, :, h0 * w.d:h1 * w.d].contiguous().to(dev)}
    del x
    dm = tsa.dims(d["Q"], d["K"])
    ws = tsa.workspace(dm, w.q, device=dev)
    Y = torch.empty_like(d["X"])
    st = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        shard.sharded_layer(d["Q"], d["K"], d["V"], d["X"], Y, q=w.q, tau=w.tau, group=group,
                            ws=ws)
    torch.cuda.synchronize(dev)
    dist.barrier()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        a.record(st)
        for _ in range(args.steps):
            _, out = shard.sharded_layer(d["Q"], d["K"], d["V"], d["X"], Y, q=w.q, tau=w.tau,
                                         group=group, ws=ws)
        b.record(st)
        torch.cuda.synchronize(dev)
        dist.barrier()
    ms = job_max(a.elapsed_time(b) / args.steps, world, dev)
    if tsa.tsa_get_device_status(ws) != 0:
        raise RuntimeError("device error in the sharded layer")
    lk = int(out["Lkeep"].item())
    lks = [torch.zeros(1, dtype=torch.int64, device=dev) for _ in range(world)]
    dist.all_gather(lks, torch.tensor([lk], dtype=torch.int64, device=dev))
    flops = 2.0 * w.H * w.d * lk * (lk + 1)
    if rank == 0:
        print(json.dumps({
            "metric": METRIC + " (one layer sharded by KV group)", "value": ms, "unit": "ms",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": False, "scaling": "strong", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": _workload_desc(w, L), "global_batch": 1, "seq_len": L,
                       "parallelism": "kv-group shard over %d rank(s): %d query heads and "
                                      "%d KV heads per rank (rank 0)" % (world, h1 - h0, kv1 - kv0),
                       "exchange": "one all-gather of 4*L bytes of partial layer score per rank"},
            "Lkeep_per_rank": [int(t.item()) for t in lks],
            "layer_tflops": flops / (ms * 1e-3) / 1e12,
            "clocks": clk.summary()}), flush=True)
    if world == 1:
        dist.destroy_process_group()


def run_score_only(args, w, L):
    """The scoring kernel alone (tsa_score: s_h and the layer score) on the workload's Q
    and K, each launch after an L2 flush that leaves L2 clean; one JSON line with the HBM
    roofline by algorithmic bytes.  Allocates only Q, K, s_h, s_l and the workspace, so a
    profiler capture of it stays small."""
    import torch

    from token_sparse_attention_dtc_b200 import tsa
    from token_sparse_attention_dtc_b200.inputs import make_workload

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    x = make_workload(w.name, seed=args.seed, L=L, B=1)
    Q, K = x["Q"].to(dev), x["K"].to(dev)
    del x
    dm = tsa.dims(Q, K)
    ws = tsa.workspace(dm, w.q, device=dev)
    s_h = torch.empty(1, w.H, L, device=dev)
    s_l = torch.empty(1, L, device=dev)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    st = torch.cuda.current_stream(dev)
    for _ in range(max(args.warmup, 3)):
        tsa.tsa_score(Q, K, w.q, s_h=s_h, s_l=s_l, ws=ws)
    ts = []
    for _ in range(args.steps):
        flush.zero_()
        flush.view(torch.int32).max()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(st)
        tsa.tsa_score(Q, K, w.q, s_h=s_h, s_l=s_l, ws=ws)
        b.record(st)
        b.synchronize()
        ts.append(a.elapsed_time(b))
    if tsa.tsa_get_device_status(ws) != 0:
        raise RuntimeError("device error in the scoring runs")
    ms = statistics.median(ts)
    nbytes = L * w.Hkv * w.d * 2 + w.q * w.H * w.d * 2 + 4 * w.H * L + 4 * L
    pk = _peaks()
    kern = score_kernel_name(args.score_schedule, w, L)
    print(json.dumps({
        "metric": "scoring kernel ms (tsa_score: s_h and s_l)", "value": ms, "unit": "ms",
        "higher_is_better": False, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": _workload_desc(w, L), "score_kernel": kern,
                   "l2": "L2 flushed (512 MB written, then read) before each launch"},
        "roofline": {"bound": "hbm", "achieved": nbytes / (ms * 1e-3) / 1e9, "peak": pk["hbm"],
                     "unit": "GB/s", "frac": nbytes / (ms * 1e-3) / 1e9 / pk["hbm"],
                     "traffic": _traffic(kern, _traffic_key(w, L)),
                     "algorithmic_bytes": nbytes}}),
          flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=("ours", "reference"))
    ap.add_argument("--workload", default="llama8b_128k")
    ap.add_argument("--L", type=int, default=None)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-attn-seconds", type=float, default=30.0,
                    help="host-core seconds of oracle attention in the cpu_baseline leg")
    ap.add_argument("--ref-attn-seconds", type=float, default=3.0,
                    help="host-core seconds of oracle attention per --impl reference step")
    ap.add_argument("--no-pages-sparsity", action="store_true")
    ap.add_argument("--stack", action="store_true",
                    help="32-layer stack with the sparse set chosen by the drift pass")
    ap.add_argument("--sweep", action="store_true", help="tau x q sweep, B = 2, L = 64K")
    ap.add_argument("--parallel", default="replicas", choices=("replicas", "kv"),
                    help="N > 1: independent layers per rank (default), or one layer "
                         "sharded by KV group across the ranks")
    ap.add_argument("--score-only", action="store_true",
                    help="time the scoring kernel alone on the workload (L2 flushed per launch)")
    ap.add_argument("--drift", action="store_true",
                    help="drift pass on 32-layer Llama-8B-shaped calibration states")
    ap.add_argument("--score-schedule", default="auto", choices=("auto", "single", "wave"),
                    help="bf16 scoring kernel: the library's automatic choice (default), the "
                         "single-wave kernel everywhere, or the wave-scheduled kernel")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3) if args.impl == "ours" else args.warmup

    from token_sparse_attention_dtc_b200.inputs import WORKLOADS

    w = WORKLOADS[args.workload]
    L = args.L or w.L
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.stack:
        run_stack(args, args.L or 4096)
        return
    if args.sweep:
        run_sweep(args)
        return
    if args.drift:
        run_drift(args)
        return
    if args.impl == "reference":  # rank 0 alone times the oracle; other ranks exit
        run_reference(args, w, L, rank, world)
        return
    if args.score_schedule != "auto":
        from token_sparse_attention_dtc_b200 import tsa

        tsa.tsa_set_score_schedule(1 if args.score_schedule == "wave" else "single", 0)
    if args.score_only:
        run_score_only(args, w, L)
        return
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        if args.parallel == "kv":
            run_kv_shard(args, w, L, rank, world, local_rank)
        else:
            run_ours(args, w, L, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
