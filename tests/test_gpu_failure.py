"""Failure detection on the GPU, without faulting it.

Every device-side wait in the tensor-core kernels is bounded in time.  The test hook
tsa_set_test_stall makes each kernel's MMA issuer wait on a barrier that nothing
completes; with a 20 ms limit that wait runs out, and the kernel must record
TSA_ERR_DEVICE_TIMEOUT in the workspace, finish the copies and MMAs it started, free its
tensor memory and exit.  The host reads the status, and the same context must then run
the next launch correctly.
"""
import pytest
import torch

from token_sparse_attention_dtc_b200 import tsa
from token_sparse_attention_dtc_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu

DEFAULT_LIMIT_US = 2_000_000
TIMEOUT = 6


class stalled:
    """Context: the test hook on, with a 20 ms wait limit."""

    def __enter__(self):
        tsa.tsa_set_wait_limit(20_000)
        tsa.tsa_set_test_stall(True)

    def __exit__(self, *a):
        tsa.tsa_set_test_stall(False)
        tsa.tsa_set_wait_limit(DEFAULT_LIMIT_US)


def _stage_inputs():
    x = make_inputs(1, 1000, 8, 2, 128, torch.bfloat16, seed=31)
    d = {k: v.cuda() for k, v in x.items()}
    dm = tsa.dims(d["Q"], d["K"])
    ws = tsa.workspace(dm, 16)
    s_h, s_l = tsa.tsa_score(d["Q"], d["K"], 16, ws=ws)
    Lk = tsa.tsa_budget(dm, s_l, 0.02, ws=ws)
    idx = tsa.tsa_select(dm, s_h, Lk, ws=ws)
    Qh, Kh, Vh = tsa.tsa_gather_qkv(d["Q"], d["K"], d["V"], idx, Lk, ws=ws)
    assert tsa.tsa_get_device_status(ws) == 0
    return d, dm, Lk, Qh, Kh, Vh, s_h, s_l


def test_attention_wait_timeout_is_reported_and_context_recovers():
    d, dm, Lk, Qh, Kh, Vh, _, _ = _stage_inputs()
    lk = int(Lk.item())
    ref = tsa.tsa_attn(dm, Qh, Kh, Vh, Lk)[:, :, :lk].clone()
    ws = tsa.workspace(dm, 16)
    with stalled():
        tsa.tsa_attn(dm, Qh, Kh, Vh, Lk, ws=ws)
        st = tsa.tsa_get_device_status(ws)
    assert st == TIMEOUT
    assert tsa.tsa_get_device_status(ws) == 0  # reading the status clears it
    again = tsa.tsa_attn(dm, Qh, Kh, Vh, Lk, ws=ws)[:, :, :lk]
    assert tsa.tsa_get_device_status(ws) == 0
    assert torch.equal(again, ref)
    # the dense mode goes through the same waits
    with stalled():
        tsa.tsa_attn(dm, d["Q"], d["K"], d["V"], None, dense=True, ws=ws)
        st = tsa.tsa_get_device_status(ws)
    assert st == TIMEOUT


@pytest.mark.parametrize("wave", [True, False])
def test_scoring_wait_timeout_is_reported_and_context_recovers(wave):
    """Both scoring kernels (the single-wave default and the wave-scheduled one, which
    this shape takes when asked) time out, report it, and score correctly afterwards."""
    d, dm, _, _, _, _, s_h_ref, s_l_ref = _stage_inputs()
    ws = tsa.workspace(dm, 16)
    tsa.tsa_set_score_schedule(wave, 0)
    try:
        with stalled():
            tsa.tsa_score(d["Q"], d["K"], 16, ws=ws)
            st = tsa.tsa_get_device_status(ws)
        assert st == TIMEOUT
        s_h, s_l = tsa.tsa_score(d["Q"], d["K"], 16, ws=ws)
        assert tsa.tsa_get_device_status(ws) == 0
    finally:
        tsa.tsa_set_score_schedule(False, 0)
    if not wave:
        assert torch.equal(s_h, s_h_ref) and torch.equal(s_l, s_l_ref)
    else:  # the reference scores came from the default (single-wave) kernel
        torch.testing.assert_close(s_h, s_h_ref, rtol=1e-5, atol=1e-30)
        torch.testing.assert_close(s_l, s_l_ref, rtol=1e-5, atol=1e-30)


def test_one_wave_scoring_wait_timeout_is_reported_and_context_recovers():
    """The automatic one-wave schedule (K of at least 192 MiB: 98304 tokens of the Llama
    shape) times out the same way.  Its grid barrier and counters reset themselves at the
    end of every launch, the timed-out one included, so the next launches give the first
    launch's scores bit for bit."""
    x = make_inputs(1, 98304, 32, 8, 128, torch.bfloat16, seed=41)
    Q, K = x["Q"].cuda(), x["K"].cuda()
    del x
    dm = tsa.dims(Q, K)
    ws = tsa.workspace(dm, 16)
    ref_h, ref_l = (t.clone() for t in tsa.tsa_score(Q, K, 16, ws=ws))
    assert tsa.tsa_get_device_status(ws) == 0
    with stalled():
        tsa.tsa_score(Q, K, 16, ws=ws)
        st = tsa.tsa_get_device_status(ws)
    assert st == TIMEOUT
    for _ in range(2):
        s_h, s_l = tsa.tsa_score(Q, K, 16, ws=ws)
        assert tsa.tsa_get_device_status(ws) == 0
        assert torch.equal(s_h, ref_h) and torch.equal(s_l, ref_l)


def test_out_of_range_scores_are_flagged():
    """The budget and selection flag scores outside their legal range (NaN, < 0, or a
    layer score above 1) instead of using them silently."""
    dm = tsa.Dims(1, 4096, 2, 1, 64, tsa.TSA_BF16)
    ws = tsa.workspace(dm, 1)
    s = torch.full((1, 4096), 1.0 / 4096, device="cuda")
    s[0, 17] = float("nan")
    tsa.tsa_budget(dm, s, 0.01, ws=ws)
    assert tsa.tsa_get_device_status(ws) == 7
    sh = torch.rand(1, 2, 4096, device="cuda")
    sh[0, 1, 5] = -1.0
    tsa.tsa_select(dm, sh, torch.tensor([100], dtype=torch.int32, device="cuda"), ws=ws)
    assert tsa.tsa_get_device_status(ws) == 7
    # in-range scores give no error
    tsa.tsa_budget(dm, torch.full((1, 4096), 1.0 / 4096, device="cuda"), 0.01, ws=ws)
    assert tsa.tsa_get_device_status(ws) == 0


def test_direct_gather_and_block_modes_time_out_and_recover():
    """The cp.async producer of the direct-gather mode and the mask walk of the block mode
    go through the same bounded waits."""
    d, dm, Lk, Qh, Kh, Vh, s_h, _ = _stage_inputs()
    idx = tsa.tsa_select(dm, s_h, Lk)
    ws = tsa.workspace(dm, 16)
    want_y = tsa.tsa_attn_gather(d["Q"], d["K"], d["V"], idx, Lk, d["X"], ws=ws)
    _, mask = tsa.tsa_block_select(dm, Qh, Kh, Lk, 0.5, logits=False)
    want_o = tsa.tsa_attn_block(dm, Qh, Kh, Vh, Lk, mask, ws=ws)
    lk = int(Lk.item())
    assert tsa.tsa_get_device_status(ws) == 0
    with stalled():
        tsa.tsa_attn_gather(d["Q"], d["K"], d["V"], idx, Lk, d["X"], ws=ws)
        st_g = tsa.tsa_get_device_status(ws)
        tsa.tsa_attn_block(dm, Qh, Kh, Vh, Lk, mask, ws=ws)
        st_b = tsa.tsa_get_device_status(ws)
    assert st_g == TIMEOUT and st_b == TIMEOUT
    assert torch.equal(tsa.tsa_attn_gather(d["Q"], d["K"], d["V"], idx, Lk, d["X"], ws=ws), want_y)
    got_o = tsa.tsa_attn_block(dm, Qh, Kh, Vh, Lk, mask, ws=ws)
    assert torch.equal(got_o[:, :, :lk], want_o[:, :, :lk])
    assert tsa.tsa_get_device_status(ws) == 0
