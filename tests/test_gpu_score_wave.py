"""The two tensor-core scoring kernels against the oracle, through the C ABI.

The wave-scheduled kernel scores the KV groups in waves (pass 1 of wave w+1 runs before
pass 2 of wave w; each CTA merges its group's statistics after a per-wave count); the
single-wave kernel scores every group at once.  The automatic schedule (the default)
takes the wave-scheduled kernel with every group in one wave when K holds at least
192 MiB, and the single-wave kernel below.  Every kernel and plan must give s_h and s_l within the
scoring tolerance (relative 1e-5) of the oracle on the same inputs, on shapes that cover:
- one wave, two waves, and many waves (the two statistics slots reused);
- a ragged last tile, the shortest eligible sequence (16 tokens, one tile), and a tile
  holding a single token;
- 1, 2 and 4 query heads per KV head (idle epilogue warps when fewer than 4);
- d = 64 and 128, batches of 1 to 20 sequences (160 KV groups in one launch);
- the automatic one-wave plan with 201 and 268 MB of K (a ragged tail, and two
  sequences).
"""
import numpy as np
import pytest
import torch

import oracle
from token_sparse_attention_dtc_b200 import tsa
from token_sparse_attention_dtc_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu


def _close(gpu, ref, what):
    gpu = np.asarray(gpu, np.float64)
    err = np.abs(gpu - ref) / np.maximum(np.abs(ref), 1e-30)
    worst = np.unravel_index(np.argmax(err), err.shape)
    assert err.max() <= 1e-5, "%s: rel err %.3g at %s (gpu %r ref %r)" % (
        what, err.max(), worst, gpu[worst], ref[worst])


class schedule:
    def __init__(self, wave, cap=0):
        self.wave, self.cap = wave, cap

    def __enter__(self):
        tsa.tsa_set_score_schedule(self.wave, self.cap)

    def __exit__(self, *a):
        tsa.tsa_set_score_schedule(0, 0)  # the default: automatic


# (B, L, H, Hkv, d, groups-per-wave cap): the comment gives the wave plan on 148 SMs
CASES = [
    (1, 4096, 32, 8, 128, 0),   # 2 waves of 4 groups, 32 CTAs per group (a tile each)
    (1, 4096, 32, 8, 128, 1),   # 8 waves of one group: each statistics slot used 4 times
    (2, 1500, 8, 2, 64, 0),     # ragged last tile (1500 = 11 * 128 + 92), 2 waves
    (3, 777, 6, 3, 128, 3),     # 2 heads per KV head, 3 waves of 3 groups
    (1, 16, 4, 1, 128, 0),      # 16 tokens: one wave, one CTA, one tile
    (1, 200, 4, 4, 64, 1),      # one head per KV head, 4 waves
    (2, 129, 4, 2, 128, 0),     # the second tile holds one token
    (20, 200, 16, 8, 64, 0),    # 160 KV groups, one launch (2 waves of 80)
]


@pytest.mark.parametrize("B,L,H,Hkv,d,cap", CASES)
def test_wave_and_single_wave_scoring_match_the_oracle(B, L, H, Hkv, d, cap):
    x = make_inputs(B, L, H, Hkv, d, torch.bfloat16, seed=B * 1000 + L + H)
    Q, K = x["Q"].cuda(), x["K"].cuda()
    ref_h, ref_l = oracle.score(x["Q"], x["K"], 16)
    out = {}
    for wave in (True, "single"):
        with schedule(wave, cap):
            s_h, s_l = tsa.tsa_score(Q, K, 16)
            torch.cuda.synchronize()
        _close(s_h.cpu().numpy(), ref_h, "s_h wave=%s" % wave)
        _close(s_l.cpu().numpy(), ref_l, "s_l wave=%s" % wave)
        out[wave] = (s_h, s_l)
    # the two schedules agree with each other to fp32 summation order
    for a, b in zip(out[True], out["single"]):
        np.testing.assert_allclose(a.cpu().numpy(), b.cpu().numpy(), rtol=1e-5, atol=1e-30)


def test_wave_scoring_is_deterministic_across_launches_and_wave_counts():
    """Repeated launches give identical bits; so do the per-wave merges, whatever the
    arrival order of the CTAs (the last one merges every CTA's pairs in split order)."""
    x = make_inputs(2, 3000, 16, 4, 128, torch.bfloat16, seed=77)
    Q, K = x["Q"].cuda(), x["K"].cuda()
    for cap in (0, 1):
        with schedule(True, cap):
            ref = tsa.tsa_score(Q, K, 16)
            for _ in range(5):
                s_h, s_l = tsa.tsa_score(Q, K, 16)
                assert torch.equal(s_h, ref[0]) and torch.equal(s_l, ref[1])


def test_wave_scoring_inside_a_layer_matches_the_oracle():
    """tsa_layer runs the same scoring launch (layer score fused): its s_h and s_l equal
    the oracle's too, here with 2 waves of one KV group."""
    x = make_inputs(1, 2048, 8, 2, 128, torch.bfloat16, seed=91)
    d = {k: v.cuda() for k, v in x.items()}
    s_h = torch.empty(1, 8, 2048, device="cuda")
    s_l = torch.empty(1, 2048, device="cuda")
    with schedule(True, 1):
        tsa.tsa_layer(d["Q"], d["K"], d["V"], d["X"], q=16, tau=0.01, s_h=s_h, s_l=s_l)
        torch.cuda.synchronize()
    ref_h, ref_l = oracle.score(x["Q"], x["K"], 16)
    _close(s_h.cpu().numpy(), ref_h, "s_h in a layer")
    _close(s_l.cpu().numpy(), ref_l, "s_l in a layer")


@pytest.mark.parametrize("B,L,H,Hkv", [(1, 98304 + 37, 32, 8), (2, 65536, 32, 8)])
def test_automatic_one_wave_schedule_matches_the_oracle(B, L, H, Hkv):
    """With at least 192 MiB of K the default schedule scores every KV group in one wave
    of the wave-scheduled kernel (here 201 and 268 MB); it matches the oracle and the
    single-wave kernel, and repeated launches are bit-identical."""
    x = make_inputs(B, L, H, Hkv, 128, torch.bfloat16, seed=L + B)
    Q, K = x["Q"].cuda(), x["K"].cuda()
    ref_h, ref_l = oracle.score(x["Q"], x["K"], 16)
    s_h, s_l = tsa.tsa_score(Q, K, 16)                  # automatic
    _close(s_h.cpu().numpy(), ref_h, "s_h one wave")
    _close(s_l.cpu().numpy(), ref_l, "s_l one wave")
    again = tsa.tsa_score(Q, K, 16)
    assert torch.equal(again[0], s_h) and torch.equal(again[1], s_l)
    with schedule("single"):
        u_h, u_l = tsa.tsa_score(Q, K, 16)
    _close(u_h.cpu().numpy(), ref_h, "s_h single wave")
    np.testing.assert_allclose(s_l.cpu().numpy(), u_l.cpu().numpy(), rtol=1e-5, atol=1e-30)
