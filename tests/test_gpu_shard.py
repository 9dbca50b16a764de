"""One layer sharded by KV group, run on one GPU as its shards in sequence.

Each shard holds a contiguous range of KV groups (their query heads' Q, their K and V,
and their columns of X).  tsa_score_partial gives each shard's s_h and unnormalised
partial layer score; tsa_layer_score_combine sums the partials in shard order and
normalises.  Checked against the oracle on the unsharded layer:
  * s_h of every shard and the combined s_l: relative 1e-5 (absolute floor 1e-30);
  * L' bit-exact against the oracle's budget re-run on the GPU's combined s_l, and
    each shard's index lists bit-exact against the oracle's selection on its s_h;
  * each shard's columns of Y against X + the oracle's attention on those indices
    (2e-2 plus half a bf16 ulp), unselected segments bitwise X;
  * the combination is deterministic, and sharded_layer (the torch.distributed driver,
    here with a single rank) agrees with the staged single-GPU layer.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
from token_sparse_attention_dtc_b200 import shard, tsa
from token_sparse_attention_dtc_b200.inputs import make_inputs

from test_gpu_parity import assert_scores_close
from test_gpu_variants import _check_y

pytestmark = pytest.mark.gpu


def _cut(x, h0, h1, kv0, kv1):
    d = x["Q"].shape[3]
    return dict(Q=x["Q"][:, :, h0:h1].contiguous(), K=x["K"][:, :, kv0:kv1].contiguous(),
                V=x["V"][:, :, kv0:kv1].contiguous(),
                X=x["X"][:, :, h0 * d:h1 * d].contiguous())


@pytest.mark.parametrize("B,L,H,Hkv,world,q,tau", [(1, 4096, 32, 8, 2, 16, 0.005),
                                                    (2, 1500, 32, 8, 4, 16, 0.02),
                                                    (1, 3000, 8, 4, 3, 64, 0.01)])
def test_sharded_layer_matches_oracle(B, L, H, Hkv, world, q, tau):
    x = make_inputs(B, L, H, Hkv, 128, torch.bfloat16, seed=L + world)
    shards = []
    for r in range(world):
        h0, h1 = shard.head_range(H, Hkv, r, world)
        kv0, kv1 = shard.kv_group_range(Hkv, r, world)
        xs = _cut(x, h0, h1, kv0, kv1)
        d = {k: v.cuda() for k, v in xs.items()}
        s_h, u = tsa.tsa_score_partial(d["Q"], d["K"], q)
        shards.append(dict(x=xs, d=d, h=(h0, h1), s_h=s_h, u=u))
    parts = torch.stack([s["u"] for s in shards])
    dm = tsa.dims(shards[0]["d"]["Q"], shards[0]["d"]["K"])
    s_l = tsa.tsa_layer_score_combine(dm, parts)
    assert torch.equal(s_l, tsa.tsa_layer_score_combine(dm, parts.clone()))
    ref_h, ref_l = oracle.score(x["Q"], x["K"], q)
    g_sl = s_l.cpu().numpy()
    assert_scores_close(g_sl, ref_l, "combined s_l")
    lk, _ = oracle.budget(g_sl, tau)
    for s in shards:
        h0, h1 = s["h"]
        d = s["d"]
        g_sh = s["s_h"].cpu().numpy()
        assert_scores_close(g_sh, ref_h[:, h0:h1], "s_h of heads %d-%d" % (h0, h1))
        sdm = tsa.dims(d["Q"], d["K"])
        Lk = tsa.tsa_budget(sdm, s_l, tau)       # every shard derives the same budget
        np.testing.assert_array_equal(Lk.cpu().numpy(), lk)
        idx = tsa.tsa_select(sdm, s["s_h"], Lk)
        ref_idx = oracle.select(g_sh, lk)
        np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)
        Qh, Kh, Vh = tsa.tsa_gather_qkv(d["Q"], d["K"], d["V"], idx, Lk)
        Oh = tsa.tsa_attn(sdm, Qh, Kh, Vh, Lk)
        Y = tsa.tsa_scatter_residual(sdm, Oh, idx, Lk, d["X"])
        _check_y(s["x"], ref_idx, lk, Y.cpu())


def test_sharded_layer_driver_single_rank_equals_the_stages():
    """shard.sharded_layer through torch.distributed (NCCL, one rank: the exchange is the
    identity): s_h bit for bit and s_l within the score tolerance of tsa_score's (the
    layer total is summed in another order), L' bit-exact against the oracle's budget
    on its s_l, and, when L' equals the staged layer's, the same indices and Y."""
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1)
    try:
        x = make_inputs(1, 2000, 32, 8, 128, torch.bfloat16, seed=3)
        d = {k: v.cuda() for k, v in x.items()}
        Y, out = shard.sharded_layer(d["Q"], d["K"], d["V"], d["X"], q=16, tau=0.01)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    dm = tsa.dims(d["Q"], d["K"])
    s_h, s_l = tsa.tsa_score(d["Q"], d["K"], 16)
    lk = tsa.tsa_budget(dm, s_l, 0.01)
    idx = tsa.tsa_select(dm, s_h, lk)
    Qh, Kh, Vh = tsa.tsa_gather_qkv(d["Q"], d["K"], d["V"], idx, lk)
    Y2 = tsa.tsa_scatter_residual(dm, tsa.tsa_attn(dm, Qh, Kh, Vh, lk), idx, lk, d["X"])
    assert torch.equal(out["s_h"], s_h)
    assert_scores_close(out["s_l"].cpu().numpy(), s_l.cpu().double().numpy(), "s_l")
    if torch.equal(out["Lkeep"], lk):
        assert torch.equal(out["idx"], idx) and torch.equal(Y, Y2)
    ref_lk, _ = oracle.budget(out["s_l"].cpu().numpy(), 0.01)
    np.testing.assert_array_equal(out["Lkeep"].cpu().numpy(), ref_lk)
