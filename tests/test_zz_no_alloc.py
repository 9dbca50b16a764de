"""tsa_score_fixed_scratch: scoring for callers that cannot allocate device memory at
call time (an engine whose device memory is planned up front by its own allocator, or a
host thread that must not enter the CUDA allocator).  It must give tsa_score's results
from its fixed device scratch, call after call, and refuse sizes the scratch cannot hold.

This file is collected last on purpose, so that a run stopping at its first failure
has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from token_sparse_attention_dtc_b200 import tsa
from token_sparse_attention_dtc_b200.inputs import make_inputs, make_workload


def _close(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    rel = np.abs(a - b) / np.maximum(np.abs(b), 1e-30)
    return rel.max() <= 1e-5


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
    cases = [make_workload("llama8b_4k", seed=11),
             make_inputs(2, 1000, 8, 2, 64, torch.bfloat16, seed=12)]
    for x in cases:  # two calls in a row, different shapes: stale scratch must not matter
        Q, K = x["Q"].cuda(), x["K"].cuda()
        ref_h, ref_l = tsa.tsa_score(Q, K, 16)
        got_h, got_l = tsa.tsa_score_fixed_scratch(Q, K, 16)
        torch.cuda.synchronize()
        assert _close(got_h, ref_h) and _close(got_l, ref_l)
    # and the same call again on the first case
    x = cases[0]
    Q, K = x["Q"].cuda(), x["K"].cuda()
    ref_h, ref_l = tsa.tsa_score(Q, K, 16)
    got_h, got_l = tsa.tsa_score_fixed_scratch(Q, K, 16)
    torch.cuda.synchronize()
    assert _close(got_h, ref_h) and _close(got_l, ref_l)
