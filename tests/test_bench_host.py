"""Host logic of bench.py on the CPU: the algorithmic work counts that the reported
rooflines divide by, the traffic lookup keyed by source hash, and the peak fallback."""
import hashlib
import json
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _mask(H, L, kept):
    """Block mask [1, H, NP, NW] int32 with bit b of (h, p) set iff kept(h, p, b)."""
    NP, NB = (L + 255) // 256, (L + 127) // 128
    NW = (NB + 31) // 32
    m = np.zeros((1, H, NP, NW), np.uint32)
    for h in range(H):
        for p in range(NP):
            for b in range(min(NB, 2 * p + 2)):
                if kept(h, p, b):
                    m[0, h, p, b // 32] |= np.uint32(1) << np.uint32(b % 32)
    return torch.from_numpy(m.view(np.int32))


def _brute_flops(mask, lk, d):
    """4 d per (query i, key j) with j <= i < lk and key block j // 128 kept for i's pair."""
    m = mask.numpy().view(np.uint32)[0]
    total = 0
    for h in range(m.shape[0]):
        for i in range(lk):
            p = i // 256
            j = np.arange(i + 1)
            b = j // 128
            total += int(((m[h, p, b // 32] >> (b % 32).astype(np.uint32)) & 1).sum())
    return 4.0 * d * total


def test_block_useful_flops_full_mask_is_the_causal_count():
    H, L, d = 2, 1000, 128
    for lk in (1000, 700, 129, 1):
        full = _mask(H, L, lambda h, p, b: True)
        assert bench.block_useful_flops(full, lk, d) == 2.0 * H * d * lk * (lk + 1)


def test_block_useful_flops_matches_brute_force_on_a_random_mask():
    rng = np.random.default_rng(3)
    H, L, d = 3, 900, 64
    keep = rng.random((H, (L + 255) // 256, 8)) < 0.5
    mask = _mask(H, L, lambda h, p, b: b >= 2 * p or b == 0 or keep[h, p, b])
    for lk in (900, 517):
        assert bench.block_useful_flops(mask, lk, d) == _brute_flops(mask, lk, d)


def test_block_useful_flops_empty_mask_counts_nothing():
    mask = _mask(2, 600, lambda h, p, b: False)
    assert bench.block_useful_flops(mask, 600, 128) == 0.0


def test_kv_union_rows_counts_each_kv_head_once_per_token():
    # 4 query heads, 2 KV heads (heads 0,1 -> group 0; heads 2,3 -> group 1), L = 8, L' = 3
    idx = torch.tensor([[[0, 1, 2, 7, 7, 7, 7, 7],
                         [1, 2, 3, 7, 7, 7, 7, 7],
                         [5, 6, 7, 0, 0, 0, 0, 0],
                         [5, 6, 7, 0, 0, 0, 0, 0]]], dtype=torch.int32)
    # group 0: {0,1,2} u {1,2,3} = 4 rows; group 1: {5,6,7} = 3 rows
    assert bench.kv_union_rows(idx, 3, 2) == 7
    assert bench.kv_union_rows(idx, 0, 2) == 0


def test_traffic_lookup_is_void_once_the_source_changes(tmp_path, monkeypatch):
    csrc = tmp_path / "token_sparse_attention_dtc_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    src = csrc / "k.cu"
    src.write_bytes(b"kernel v1\n")
    sha = hashlib.sha256(b"kernel v1\n").hexdigest()[:16]
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(
        {"k_x": {"w": {"source": "k.cu", "source_sha": sha, "bytes_per_launch": 123.0}}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench._traffic("k_x", "w") == 123.0
    assert bench._traffic("k_x", "other") is None
    assert bench._traffic("k_y", "w") is None
    src.write_bytes(b"kernel v2\n")
    assert bench._traffic("k_x", "w") is None


def test_traffic_key_applies_only_at_the_captured_length():
    """A capture keyed by a workload name stands for that workload's own length; a run with
    --L at another length reports no traffic."""
    from token_sparse_attention_dtc_b200.inputs import WORKLOADS
    w = WORKLOADS["llama8b_128k"]
    assert bench._traffic_key(w, w.L) == "llama8b_128k"
    assert bench._traffic_key(w, 98304) is None
    assert bench._traffic("k_attn_tc", None) is None


def test_peaks_read_the_measured_file_else_the_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    fb = bench._peaks()
    assert fb["src"] == "fallback" and fb["hbm"] > 0 and fb["bf16"] > fb["bf16_sus"] > 0
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps(
        {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}))
    pk = bench._peaks()
    assert pk == dict(hbm=6000.0, bf16=1600.0, bf16_sus=1400.0, src="measured")


def test_l2_note_says_whether_every_input_exceeds_l2():
    big = {k: torch.empty(64 * 2**20, dtype=torch.bfloat16, device="meta") for k in "QKVX"}
    assert bench.l2_note(big).startswith("inputs larger than L2")
    small = dict(big, K=torch.empty(10, dtype=torch.bfloat16, device="meta"))
    assert bench.l2_note(small).startswith("inputs not all larger than L2")
