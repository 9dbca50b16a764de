"""tsa_score_fixed_scratch: scoring for callers that cannot allocate device memory at
call time (an engine whose device memory is planned up front by its own allocator, or a
host thread that must not enter the CUDA allocator).  It must give tsa_score's results
from its fixed device scratch, call after call, refuse sizes the scratch cannot hold,
and report a device-side error through tsa_score_fixed_scratch_status.

This file is collected last on purpose, so that a run stopping at its first failure
has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from token_sparse_attention_dtc_b200 import tsa
from token_sparse_attention_dtc_b200.inputs import make_inputs, make_workload

TIMEOUT = 6  # TSA_ERR_DEVICE_TIMEOUT


def test_fixed_scratch_rejects_sizes_beyond_its_limit():
    # 16 sequences of 2^20 tokens need ~17 MB of scoring scratch: refused on the host,
    # before any device work (so this runs without a GPU too).
    dm = tsa.Dims(16, 1 << 20, 32, 8, 128, tsa.TSA_BF16)
    assert tsa.workspace_size(dm, 16) > (2 << 20)
    P = ctypes.c_void_p(0x10000)
    st = tsa.lib().tsa_score_fixed_scratch(ctypes.byref(dm), P, P, 16, 0.088, P, P, None)
    assert st == 4  # TSA_ERR_WORKSPACE
    assert b"fixed" in tsa.lib().tsa_last_error()


@pytest.mark.gpu
def test_fixed_scratch_matches_tsa_score_on_consecutive_calls():
    """The same kernels as tsa_score on the same inputs: bit for bit, on calls in a row
    with different shapes (stale scratch must not matter), and within the scoring
    tolerance of the oracle."""
    cases = [make_workload("llama8b_4k", seed=11),
             make_inputs(2, 1000, 8, 2, 64, torch.bfloat16, seed=12)]
    assert tsa.tsa_score_fixed_scratch_status() == 0
    for x in cases:
        Q, K = x["Q"].cuda(), x["K"].cuda()
        ref_h, ref_l = tsa.tsa_score(Q, K, 16)
        got_h, got_l = tsa.tsa_score_fixed_scratch(Q, K, 16)
        assert tsa.tsa_score_fixed_scratch_status() == 0
        assert torch.equal(got_h, ref_h) and torch.equal(got_l, ref_l)
    # the same call again on the first case, then against the oracle
    x = cases[0]
    Q, K = x["Q"].cuda(), x["K"].cuda()
    ref_h, ref_l = tsa.tsa_score(Q, K, 16)
    got_h, got_l = tsa.tsa_score_fixed_scratch(Q, K, 16)
    assert tsa.tsa_score_fixed_scratch_status() == 0
    assert torch.equal(got_h, ref_h) and torch.equal(got_l, ref_l)
    o_h, o_l = oracle.score(x["Q"], x["K"], 16)
    for got, ref in ((got_h, o_h), (got_l, o_l)):
        g = got.cpu().double().numpy()
        assert np.max(np.abs(g - ref) / np.maximum(np.abs(ref), 1e-30)) <= 1e-5


@pytest.mark.gpu
def test_fixed_scratch_one_wave_schedule_matches_tsa_score():
    """At 98304 tokens of the Llama shape (201 MB of K) the scoring takes the one-wave
    kernel, whose counters live in the fixed array too: bit for bit tsa_score's result on
    two calls in a row."""
    x = make_inputs(1, 98304, 32, 8, 128, torch.bfloat16, seed=13)
    Q, K = x["Q"].cuda(), x["K"].cuda()
    ref_h, ref_l = tsa.tsa_score(Q, K, 16)
    for _ in range(2):
        got_h, got_l = tsa.tsa_score_fixed_scratch(Q, K, 16)
        assert tsa.tsa_score_fixed_scratch_status() == 0
        assert torch.equal(got_h, ref_h) and torch.equal(got_l, ref_l)


@pytest.mark.gpu
def test_fixed_scratch_reports_a_device_timeout_and_recovers():
    """A bounded device wait that runs out (the stall test hook, 20 ms limit) is
    reported by tsa_score_fixed_scratch_status, once; the next call is exact again."""
    x = make_inputs(1, 1000, 8, 2, 128, torch.bfloat16, seed=31)
    Q, K = x["Q"].cuda(), x["K"].cuda()
    ref_h, ref_l = tsa.tsa_score(Q, K, 16)
    tsa.tsa_set_wait_limit(20_000)
    tsa.tsa_set_test_stall(True)
    try:
        tsa.tsa_score_fixed_scratch(Q, K, 16)
        st = tsa.tsa_score_fixed_scratch_status()
    finally:
        tsa.tsa_set_test_stall(False)
        tsa.tsa_set_wait_limit(2_000_000)
    assert st == TIMEOUT
    assert tsa.tsa_score_fixed_scratch_status() == 0  # reading it cleared it
    got_h, got_l = tsa.tsa_score_fixed_scratch(Q, K, 16)
    assert tsa.tsa_score_fixed_scratch_status() == 0
    assert torch.equal(got_h, ref_h) and torch.equal(got_l, ref_l)
