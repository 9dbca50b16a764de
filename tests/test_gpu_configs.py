"""Parity at the full sizes of the LLaMA-3.1-8B-shaped workloads, through tsa_layer (the
launch configuration the benchmark times): the 32K layer (B = 1, L = 32768, q = 16,
tau = 0.01) and the sweep shape (B = 2, L = 65536, q = 64, tau = 0.02, each sample with
its own budget).

What is checked, per workload:
  * every s_h and s_l against the oracle (relative 1e-5, absolute floor 1e-30);
  * L' per sample and every index list bit-exact against the oracle's budget and
    selection re-run on the GPU's fp32 scores;
  * every unselected segment of Y bitwise equal to X;
  * the kept segments of Y on all heads for a fixed set of compressed rows (the first
    and last rows, the rows on both sides of 128-row tile boundaries, the last tile's
    diagonal and random rows) against X + the oracle's attention on its own indices,
    within 2e-2 plus half a bf16 ulp of the result.
"""
import numpy as np
import pytest
import torch

import oracle
from token_sparse_attention_dtc_b200 import tsa
from token_sparse_attention_dtc_b200.inputs import make_workload

from test_gpu_parity import assert_scores_close

pytestmark = pytest.mark.gpu


def run_layer(x, q, tau):
    d = {k: v.cuda() for k, v in x.items()}
    B, L, H, _ = x["Q"].shape
    s_h = torch.empty(B, H, L, device="cuda")
    s_l = torch.empty(B, L, device="cuda")
    Lk = torch.empty(B, dtype=torch.int32, device="cuda")
    idx = torch.empty(B, H, L, dtype=torch.int32, device="cuda")
    ws = tsa.workspace(tsa.dims(d["Q"], d["K"]), q, layer=True)
    Y = tsa.tsa_layer(d["Q"], d["K"], d["V"], d["X"], q=q, tau=tau, s_h=s_h, s_l=s_l,
                      Lkeep=Lk, idx=idx, ws=ws)
    assert tsa.tsa_get_device_status(ws) == 0
    out = dict(s_h=s_h.cpu().numpy(), s_l=s_l.cpu().numpy(), Lkeep=Lk.cpu().numpy(),
               idx=idx.cpu().numpy(), Y=Y.cpu())
    del d, ws
    torch.cuda.empty_cache()
    return out


def sample_rows(lk, rng, edge, n_random):
    """Compressed rows to check for a sample with L' = lk."""
    if lk == 0:
        return []
    rows = set(range(min(edge, lk)))                        # first tile's first rows
    rows |= set(range(max(0, lk - edge), lk))               # last tile, diagonal included
    for t in (1, 2, lk // 256, lk // 128 - 1):              # both sides of tile boundaries
        for i in (128 * t - 1, 128 * t):
            if 0 <= i < lk:
                rows.add(i)
    rows |= set(rng.integers(0, lk, n_random).tolist())
    return sorted(rows)


def check_layer_sampled(x, q, tau, g, edge=64, n_random=48, seed=0):
    Q, K, V, X = x["Q"], x["K"], x["V"], x["X"]
    B, L, H, dd = Q.shape
    ref_h, ref_l = oracle.score(Q, K, q)
    assert_scores_close(g["s_h"], ref_h, "s_h")
    assert_scores_close(g["s_l"], ref_l, "s_l")
    lk, _ = oracle.budget(g["s_l"], tau)
    np.testing.assert_array_equal(g["Lkeep"], lk)
    idx = oracle.select(g["s_h"], lk)
    np.testing.assert_array_equal(g["idx"], idx)
    Y = g["Y"]
    # unselected segments: bitwise X (all heads, all tokens)
    for b in range(B):
        for h in range(H):
            seg = slice(h * dd, (h + 1) * dd)
            rest = torch.from_numpy(idx[b, h, lk[b]:].astype(np.int64))
            assert torch.equal(Y[b, rest, seg], X[b, rest, seg]), (b, h)
    # kept segments on sampled rows of every head
    rng = np.random.default_rng(seed)
    rows = []
    for b in range(B):
        rs = sample_rows(int(lk[b]), rng, edge, n_random)
        rows += [(b, h, i) for h in range(H) for i in rs]
    if not rows:
        return lk
    vals = oracle.attend_rows(Q, K, V, idx, lk, rows)
    r = np.asarray(rows)
    t = idx[r[:, 0], r[:, 1], r[:, 2]]
    bi = torch.from_numpy(r[:, 0:1].astype(np.int64))
    ti = torch.from_numpy(t[:, None].astype(np.int64))
    ci = torch.from_numpy(r[:, 1:2] * dd + np.arange(dd)[None, :])
    got = Y[bi, ti, ci].double().numpy()
    ref = X[bi, ti, ci].double().numpy() + vals
    excess = np.abs(got - ref) - (2e-2 + 2.0 ** -8 * np.abs(ref))
    assert excess.max() <= 0, "Y max excess %.3g at row %s" % (
        excess.max(), rows[int(np.argmax(excess.max(axis=1)))])
    return lk


def test_llama_32k_layer_at_full_size():
    x = make_workload("llama8b_32k", seed=0)
    g = run_layer(x, 16, 0.01)
    lk = check_layer_sampled(x, 16, 0.01, g)
    assert 0 < lk[0] <= 32768


def test_sweep_shape_two_samples_q64_at_full_size():
    x = make_workload("llama8b_64k_b2", seed=0)
    g = run_layer(x, 64, 0.02)
    lk = check_layer_sampled(x, 64, 0.02, g, edge=48, n_random=32)
    assert all(0 < v <= 65536 for v in lk)
