"""Bounds on caller-supplied counts and indices, on the GPU.

A kept count Lkeep[b] outside [0, L] is clamped to that range by every kernel that reads
it, and an index outside [0, L) is skipped by the scatter, so no row at or past L (and
no byte outside the caller's buffers) is read or written.  Each case writes into a view
of a larger buffer whose tail holds a sentinel, and checks that the tail is unchanged
and that the result equals the one for the clamped count.
"""
import pytest
import torch

from token_sparse_attention_dtc_b200 import tsa
from token_sparse_attention_dtc_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu

GUARD = 4096  # elements of sentinel after each output


def _guarded(shape, dtype, fill=7.0):
    n = 1
    for s in shape:
        n *= s
    buf = torch.full((n + GUARD,), fill, dtype=dtype, device="cuda")
    return buf, buf[:n].view(shape)


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.bfloat16, 64),
                                     (torch.float32, 64)])
def test_attention_clamps_a_kept_count_past_L(dtype, d):
    B, L, H, Hkv = 2, 1000, 4, 2
    x = make_inputs(B, L, H, Hkv, d, dtype, seed=91)
    dd = {k: v.cuda() for k, v in x.items()}
    dm = tsa.dims(dd["Q"], dd["K"])
    s_h, _ = tsa.tsa_score(dd["Q"], dd["K"], 16)
    full = torch.tensor([L, L], dtype=torch.int32, device="cuda")
    idx = tsa.tsa_select(dm, s_h, full)
    Qh, Kh, Vh = tsa.tsa_gather_qkv(dd["Q"], dd["K"], dd["V"], idx, full)
    want = tsa.tsa_attn(dm, Qh, Kh, Vh, full)
    ws = tsa.workspace(dm, 1)
    for bad in ([L + 100, L], [L + 100, 1 << 30]):
        buf, Oh = _guarded((B, H, L, d), dtype)
        tsa.tsa_attn(dm, Qh, Kh, Vh, torch.tensor(bad, dtype=torch.int32, device="cuda"),
                     Oh=Oh, ws=ws)
        st = tsa.tsa_get_device_status(ws)
        assert torch.equal(Oh, want)
        assert torch.all(buf[-GUARD:] == 7.0)
        if dtype == torch.bfloat16:  # the tensor-core kernel also reports it
            assert st == 1  # TSA_ERR_INVALID_ARG
    # a negative count keeps nothing and writes nothing
    buf, Oh = _guarded((B, H, L, d), dtype)
    tsa.tsa_attn(dm, Qh, Kh, Vh, torch.tensor([-5, 0], dtype=torch.int32, device="cuda"),
                 Oh=Oh, ws=ws)
    tsa.tsa_get_device_status(ws)
    assert torch.all(buf == 7.0)


@pytest.mark.parametrize("in_place", [True, False])
def test_scatter_skips_bad_indices_and_clamps_the_count(in_place):
    B, L, H, Hkv, d = 1, 700, 4, 2, 128
    x = make_inputs(B, L, H, Hkv, d, torch.bfloat16, seed=92)
    dd = {k: v.cuda() for k, v in x.items()}
    dm = tsa.dims(dd["Q"], dd["K"])
    Oh = torch.randn(B, H, L, d, device="cuda").to(torch.bfloat16)
    idx = torch.arange(L, dtype=torch.int32, device="cuda").repeat(B, H, 1).contiguous()
    bad = idx.clone()
    bad[0, 1, 5] = -1
    bad[0, 2, 9] = L
    bad[0, 3, 11] = 1 << 30
    ok_rows = torch.ones(B, H, L, dtype=torch.bool)
    ok_rows[0, 1, 5] = ok_rows[0, 2, 9] = ok_rows[0, 3, 11] = False
    good = torch.tensor([L], dtype=torch.int32, device="cuda")
    want = tsa.tsa_scatter_residual(dm, Oh, idx, good, dd["X"]).cpu()
    for count in ([L], [L + 50]):
        buf, Y = _guarded(tuple(dd["X"].shape), torch.bfloat16)
        if in_place:
            Y.copy_(dd["X"])
            tsa.tsa_scatter_residual(dm, Oh, bad, torch.tensor(count, dtype=torch.int32,
                                                                device="cuda"), Y, Y)
        else:
            tsa.tsa_scatter_residual(dm, Oh, bad, torch.tensor(count, dtype=torch.int32,
                                                                device="cuda"), dd["X"], Y)
        torch.cuda.synchronize()
        assert torch.all(buf[-GUARD:] == 7.0)
        got = Y.cpu()
        X = x["X"]
        for h in range(H):
            seg = slice(h * d, (h + 1) * d)
            rows = ok_rows[0, h].nonzero().flatten()
            assert torch.equal(got[0, rows, seg], want[0, rows, seg])
        # a token whose only writer was skipped keeps its old value
        for h, t in ((1, 5), (2, 9), (3, 11)):
            seg = slice(h * d, (h + 1) * d)
            expect = X[0, t, seg] if in_place else torch.full((d,), 7.0, dtype=torch.bfloat16)
            assert torch.equal(got[0, t, seg], expect)


def test_gather_clamps_a_kept_count_past_L():
    B, L, H, Hkv, d = 1, 300, 4, 2, 128
    x = make_inputs(B, L, H, Hkv, d, torch.bfloat16, seed=93)
    dd = {k: v.cuda() for k, v in x.items()}
    dm = tsa.dims(dd["Q"], dd["K"])
    idx = torch.arange(L, dtype=torch.int32, device="cuda").repeat(B, H, 1).contiguous()
    full = torch.tensor([L], dtype=torch.int32, device="cuda")
    want = tsa.tsa_gather_qkv(dd["Q"], dd["K"], dd["V"], idx, full)
    bufs = [_guarded((B, H, L, d), torch.bfloat16) for _ in range(3)]
    ws = tsa.workspace(dm, 1)
    tsa.tsa_gather_qkv(dd["Q"], dd["K"], dd["V"], idx,
                       torch.tensor([L + 77], dtype=torch.int32, device="cuda"),
                       *[v for _, v in bufs], ws=ws)
    assert tsa.tsa_get_device_status(ws) == 0
    for (buf, got), w in zip(bufs, want):
        assert torch.equal(got, w)
        assert torch.all(buf[-GUARD:] == 7.0)
