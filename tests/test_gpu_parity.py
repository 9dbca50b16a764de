"""GPU parity: every stage of the CUDA path against the CPU oracle, through the C ABI.

Tolerances (from the layer's numerics):
  * scores s_h, s_l: relative 1e-5 with an absolute floor of 1e-30 (fp32 softmax
    weights below that underflow differently than the fp64 oracle's);
  * budget L' and index lists: bit-exact when the oracle re-runs its budget and
    selection on the GPU's fp32 scores;
  * attention rows Ô: absolute 2e-2 for bf16, 1e-4 for fp32, with attention computed
    on the oracle's indices (asserted equal to the GPU's first);
  * Y = X + Decompress(Ô): the attention tolerance plus half an ulp of the output type
    (Y is rounded once more, to bf16 or fp32); unselected segments equal X bitwise.
"""
import numpy as np
import pytest
import torch

import oracle
from token_sparse_attention_dtc_b200 import tsa
from token_sparse_attention_dtc_b200.inputs import make_inputs, make_workload

pytestmark = pytest.mark.gpu

ATOL = {torch.bfloat16: 2e-2, torch.float32: 1e-4}
HALF_ULP = {torch.bfloat16: 2.0 ** -8, torch.float32: 2.0 ** -24}


def _dev(x):
    return {k: v.cuda() for k, v in x.items()}


def assert_scores_close(gpu, ref, what):
    gpu = np.asarray(gpu, np.float64)
    err = np.abs(gpu - ref) / np.maximum(np.abs(ref), 1e-30)
    worst = np.unravel_index(np.argmax(err), err.shape)
    assert err.max() <= 1e-5, "%s: rel err %.3g at %s (gpu %r ref %r)" % (
        what, err.max(), worst, gpu[worst], ref[worst])


def run_stages(x, q, tau, in_place=False, Lkeep_override=None):
    """Call every stage entry point once; return CPU copies of everything."""
    d = _dev(x)
    dm = tsa.dims(d["Q"], d["K"])
    ws = tsa.workspace(dm, q)
    s_h, s_l = tsa.tsa_score(d["Q"], d["K"], q, ws=ws)
    Lk = tsa.tsa_budget(dm, s_l, tau, ws=ws)
    if Lkeep_override is not None:
        Lk = torch.tensor(Lkeep_override, dtype=torch.int32, device="cuda")
    idx = tsa.tsa_select(dm, s_h, Lk, ws=ws)
    Qh, Kh, Vh = tsa.tsa_gather_qkv(d["Q"], d["K"], d["V"], idx, Lk, ws=ws)
    Oh = tsa.tsa_attn(dm, Qh, Kh, Vh, Lk, ws=ws)
    if in_place:
        Y = d["X"].clone()
        tsa.tsa_scatter_residual(dm, Oh, idx, Lk, Y, Y)
    else:
        Y = tsa.tsa_scatter_residual(dm, Oh, idx, Lk, d["X"])
    assert tsa.tsa_get_device_status(ws) == 0
    torch.cuda.synchronize()
    c = lambda t: t.cpu()
    return dict(s_h=c(s_h), s_l=c(s_l), Lkeep=c(Lk), idx=c(idx), Qh=c(Qh), Kh=c(Kh), Vh=c(Vh),
                Oh=c(Oh), Y=c(Y))


def check_layer(x, q, tau, g, full_attention=True, heads=None):
    """Compare a run_stages() result g with the oracle on the same inputs."""
    Q, K, V, X = x["Q"], x["K"], x["V"], x["X"]
    B, L, H, dd = Q.shape
    dt = Q.dtype
    # scores
    s_h, s_l = oracle.score(Q, K, q)
    assert_scores_close(g["s_h"].numpy(), s_h, "s_h")
    assert_scores_close(g["s_l"].numpy(), s_l, "s_l")
    # budget and selection, re-run by the oracle on the GPU's fp32 scores
    lk, _ = oracle.budget(g["s_l"].numpy(), tau)
    np.testing.assert_array_equal(g["Lkeep"].numpy(), lk)
    idx = oracle.select(g["s_h"].numpy(), lk)
    np.testing.assert_array_equal(g["idx"].numpy(), idx)
    # gather: bit-exact rows, zero padding up to the next 128-row tile
    G = H // K.shape[2]
    for b in range(B):
        for h in ([0, H - 1] if heads is None else heads):
            S = torch.from_numpy(idx[b, h, :lk[b]]).long()
            assert torch.equal(g["Qh"][b, h, :lk[b]], Q[b, S, h])
            assert torch.equal(g["Kh"][b, h, :lk[b]], K[b, S, h // G])
            assert torch.equal(g["Vh"][b, h, :lk[b]], V[b, S, h // G])
            pad = min(L, (int(lk[b]) + 127) // 128 * 128)
            assert torch.all(g["Vh"][b, h, lk[b]:pad] == 0)
    # attention on the oracle's indices
    if full_attention:
        Oh = oracle.attend(Q, K, V, idx, lk)
        rows = [(b, h, i) for b in range(B) for h in range(H) for i in range(int(lk[b]))]
    else:
        rows = [(b, h, i) for b in range(B) for h in heads for i in range(int(lk[b]))]
        vals = oracle.attend_rows(Q, K, V, idx, lk, rows)
        Oh = np.zeros((B, H, L, dd))
        r = np.asarray(rows).reshape(-1, 3)
        Oh[r[:, 0], r[:, 1], r[:, 2]] = vals
    if rows:
        r = np.asarray(rows)
        got = g["Oh"].double().numpy()[r[:, 0], r[:, 1], r[:, 2]]
        want = Oh[r[:, 0], r[:, 1], r[:, 2]]
        err = np.abs(got - want).max()
        assert err <= ATOL[dt], "attention max abs err %.3g" % err
    # decompress + residual
    O_dec, Y_ref = oracle.decompress_residual(Oh, idx, lk, X)
    Yg = g["Y"].double().numpy()
    Xd = X.double().numpy()
    hs = range(H) if full_attention else heads
    for b in range(B):
        for h in hs:
            seg = slice(h * dd, (h + 1) * dd)
            kept = idx[b, h, :lk[b]]
            rest = idx[b, h, lk[b]:]
            np.testing.assert_array_equal(Yg[b, rest, seg], Xd[b, rest, seg])
            if len(kept):
                diff = np.abs(Yg[b, kept, seg] - Y_ref[b, kept, seg])
                bound = ATOL[dt] + HALF_ULP[dt] * np.abs(Y_ref[b, kept, seg])
                assert np.all(diff <= bound), "Y max excess %.3g" % (diff - bound).max()
    # the scatter kernel itself: one fp32 add, one rounding
    Ot = torch.zeros(B, L, H * dd, dtype=torch.float32)
    for b in range(B):
        for h in range(H):
            kept = torch.from_numpy(idx[b, h, :lk[b]]).long()
            Ot[b, kept, h * dd:(h + 1) * dd] = g["Oh"][b, h, :lk[b]].float()
    assert torch.equal(g["Y"], (X.float() + Ot).to(dt))
    return lk


def test_tiny_mha_fp32_layer():
    x = make_workload("tiny_mha_1k", seed=0)
    g = run_stages(x, 16, 0.01)
    lk = check_layer(x, 16, 0.01, g)
    assert 0 < lk[0] < 1024


def test_llama_4k_bf16_layer():
    x = make_workload("llama8b_4k", seed=1)
    g = run_stages(x, 16, 0.005)
    lk = check_layer(x, 16, 0.005, g)
    assert 0 < lk[0] <= 4096


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.bfloat16, 64),
                                     (torch.float32, 64), (torch.float32, 128)])
def test_ragged_batch_two(dtype, d):
    x = make_inputs(2, 1000, 8, 2, d, dtype, seed=3, shift=2.5, heavy_frac=0.02)
    g = run_stages(x, 16, 0.02)
    check_layer(x, 16, 0.02, g)


def test_recent_queries_exceed_length():
    x = make_inputs(1, 10, 4, 2, 64, torch.bfloat16, seed=4)
    g = run_stages(x, 16, 0.05)
    check_layer(x, 16, 0.05, g)


@pytest.mark.parametrize("L", [1, 2, 129])
@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_shortest_sequences(L, dtype, d):
    """One token (the budget then prunes it: L' = 0, Y = X), two tokens, and one token past
    a full 128-row tile, with two samples."""
    x = make_inputs(2, L, 4, 2, d, dtype, seed=L)
    g = run_stages(x, 16, 0.05)
    check_layer(x, 16, 0.05, g)


def test_tau_zero_keeps_everything_and_matches_dense():
    x = make_inputs(1, 300, 4, 1, 128, torch.bfloat16, seed=5)
    g = run_stages(x, 16, 0.0)
    assert g["Lkeep"].tolist() == [300]
    check_layer(x, 16, 0.0, g)
    d = _dev(x)
    dm = tsa.dims(d["Q"], d["K"])
    O = tsa.tsa_attn(dm, d["Q"], d["K"], d["V"], None, dense=True)
    Y = tsa.tsa_scatter_residual(dm, O, None, None, d["X"])
    # tau = 0: the compressed and dense paths see the same problem
    Ohd = O.cpu().view(1, 300, 4, 128).permute(0, 2, 1, 3)
    assert (Ohd.float() - g["Oh"].float()).abs().max() <= 2e-2
    ref = oracle.attend(x["Q"], x["K"], x["V"], None, None)
    assert np.abs(Ohd.double().numpy() - ref).max() <= 2e-2
    assert torch.equal(Y.cpu(), (x["X"].float() + O.cpu().view(1, 300, 512).float()).to(torch.bfloat16))


@pytest.mark.parametrize("keep", [1, 2, 129, 511, 512])
def test_forced_budgets(keep):
    x = make_inputs(1, 512, 4, 2, 128, torch.bfloat16, seed=6)
    g = run_stages(x, 16, 0.01, Lkeep_override=[keep])
    idx = oracle.select(g["s_h"].numpy(), np.array([keep], np.int32))
    np.testing.assert_array_equal(g["idx"].numpy(), idx)
    rows = [(0, h, i) for h in range(4) for i in range(keep)]
    want = oracle.attend_rows(x["Q"], x["K"], x["V"], idx, np.array([keep], np.int32), rows)
    r = np.asarray(rows)
    got = g["Oh"].double().numpy()[r[:, 0], r[:, 1], r[:, 2]]
    assert np.abs(got - want).max() <= 2e-2
    if keep == 1:  # a single kept row attends to itself only
        for h in range(4):
            t = int(idx[0, h, 0])
            assert torch.equal(g["Oh"][0, h, 0], x["V"][0, t, h // 2])


def test_budget_zero_keeps_nothing():
    x = make_inputs(1, 256, 4, 2, 64, torch.bfloat16, seed=7)
    g = run_stages(x, 16, 0.01, Lkeep_override=[0])
    assert torch.equal(g["Y"], x["X"])
    assert torch.equal(g["idx"][0, 0], torch.arange(256, dtype=torch.int32))


def test_in_place_residual_matches_out_of_place():
    x = make_inputs(1, 700, 8, 2, 128, torch.bfloat16, seed=8)
    a = run_stages(x, 16, 0.01)
    b = run_stages(x, 16, 0.01, in_place=True)
    assert torch.equal(a["Y"], b["Y"])


def test_budget_synthetic_scores_bitexact():
    rng = np.random.default_rng(0)
    cases = []
    L = 5000
    cases.append(np.full(L, 1.0 / 4096, np.float32)[:4096])               # uniform 2^-12
    v = (rng.random(L) ** 4).astype(np.float32)
    cases.append((v / v.sum()).astype(np.float32))
    cases.append(np.concatenate([np.full(4, 0.25, np.float32), np.zeros(L - 4, np.float32)]))
    cases.append(np.zeros(L, np.float32))                                   # never reached
    # powers of two from 2^-13 down to subnormals: masses below one unit, exact, shifted
    w = np.ldexp(np.float32(1.0), -rng.integers(13, 150, size=L)).astype(np.float32)
    w[::7] *= np.float32(1.75)
    cases.append(w)
    for s in cases:
        for tau in (0.0, 1e-12, 0.001, 0.01, 0.25, 0.5, 0.999):
            dm = tsa.Dims(1, len(s), 1, 1, 64, tsa.TSA_BF16)
            sl = torch.from_numpy(s).cuda().view(1, -1)
            lk = tsa.tsa_budget(dm, sl, tau)
            want, _ = oracle.budget(s[None], tau)
            assert lk.cpu().numpy()[0] == want[0], (tau, s[:4])


def test_select_heavy_ties_bitexact():
    rng = np.random.default_rng(1)
    B, H, L = 2, 3, 3000
    s = (rng.integers(0, 5, size=(B, H, L)) / 8).astype(np.float32)
    for keeps in ([1, 2999], [1500, 3000], [0, 7], [2999, 1]):
        lk = np.array(keeps, np.int32)
        dm = tsa.Dims(B, L, H, 1, 64, tsa.TSA_BF16)
        idx = tsa.tsa_select(dm, torch.from_numpy(s).cuda(), torch.from_numpy(lk).cuda())
        np.testing.assert_array_equal(idx.cpu().numpy(), oracle.select(s, lk))


def test_select_multichunk_ties_bitexact():
    """Several 4096-token chunks plus a ragged tail: tied runs at the threshold cross chunk
    boundaries, keys span every digit range (zeros, denormals, values near the float
    maximum), and one row is all-equal."""
    rng = np.random.default_rng(7)
    B, H, L = 2, 4, 3 * 4096 + 517
    s = (rng.integers(0, 6, size=(B, H, L)) / 8).astype(np.float32)
    s[0, 1] = np.float32(0.375)                                        # all equal
    s[0, 2] = rng.choice(np.array([0.0, 1e-45, 1e-40, 1e-20, 1.0, 3e38], np.float32),
                         size=L)
    s[1, 3, 4000:4200] = np.float32(2.5)                               # run over a boundary
    for keeps in ([1, L - 1], [L // 2, 4095], [4096, 4097], [4100, 8192], [L, 0],
                  [rng.integers(1, L), rng.integers(1, L)]):
        lk = np.array(keeps, np.int32)
        dm = tsa.Dims(B, L, H, 1, 64, tsa.TSA_BF16)
        idx = tsa.tsa_select(dm, torch.from_numpy(s).cuda(), torch.from_numpy(lk).cuda())
        np.testing.assert_array_equal(idx.cpu().numpy(), oracle.select(s, lk), err_msg=str(keeps))


@pytest.mark.parametrize("L", [4099, 40001, 70001, 200003, 262144, 262147])
def test_budget_and_select_every_cluster_size_bitexact(L):
    """Rows of up to 8 x 32768 scores run budget and selection in one thread-block cluster
    of 1, 2, 4 or 8 CTAs (here 1, 2, 4, 8, 8); 262147 tokens take the grid-wide kernels.
    Both equal the oracle bit for bit, with heavy ties, ragged slices and a tied run that
    crosses the slices."""
    rng = np.random.default_rng(L)
    B, H = 2, 3
    s = (rng.integers(0, 7, size=(B, H, L)) / 8).astype(np.float32)
    s[1, 2, : L // 2] = np.float32(0.5)
    s[0, 1] = rng.choice(np.array([0.0, 1e-45, 1e-30, 0.25, 1.0, 3e38], np.float32), size=L)
    dm = tsa.Dims(B, L, H, 1, 64, tsa.TSA_BF16)
    s_d = torch.from_numpy(s).cuda()
    for keeps in ([int(rng.integers(1, L)), L // 2], [1, L - 1], [L, 0]):
        lk = np.array(keeps, np.int32)
        idx = tsa.tsa_select(dm, s_d, torch.from_numpy(lk).cuda())
        np.testing.assert_array_equal(idx.cpu().numpy(), oracle.select(s, lk), err_msg=str(keeps))
    v = (rng.random((B, L)) ** 4).astype(np.float32)
    sl = (v / v.sum(1, keepdims=True)).astype(np.float32)
    sl[1, 1000:3000] = np.float32(1.0 / L)
    sl_d = torch.from_numpy(sl).cuda()
    for tau in (0.0, 1e-4, 0.01, 0.3, 0.999):
        lk = tsa.tsa_budget(dm, sl_d, tau)
        want, _ = oracle.budget(sl, tau)
        np.testing.assert_array_equal(lk.cpu().numpy(), want, err_msg=str(tau))
    zero = torch.zeros(B, L, device="cuda")
    assert tsa.tsa_budget(dm, zero, 0.01).cpu().tolist() == [0, 0]  # tau never reached


def test_dense_attention_gqa_matches_oracle():
    x = make_inputs(2, 333, 8, 2, 128, torch.bfloat16, seed=9)
    d = _dev(x)
    dm = tsa.dims(d["Q"], d["K"])
    O = tsa.tsa_attn(dm, d["Q"], d["K"], d["V"], None, dense=True).cpu()
    ref = oracle.attend(x["Q"], x["K"], x["V"], None, None)          # [B,H,L,d]
    got = O.view(2, 333, 8, 128).permute(0, 2, 1, 3).double().numpy()
    assert np.abs(got - ref).max() <= 2e-2


def test_layer_entry_matches_stages():
    x = make_workload("llama8b_4k", seed=2)
    d = _dev(x)
    g = run_stages(x, 16, 0.005)
    s_h = torch.empty(1, 32, 4096, device="cuda")
    s_l = torch.empty(1, 4096, device="cuda")
    Lk = torch.empty(1, dtype=torch.int32, device="cuda")
    idx = torch.empty(1, 32, 4096, dtype=torch.int32, device="cuda")
    Y = tsa.tsa_layer(d["Q"], d["K"], d["V"], d["X"], q=16, tau=0.005, s_h=s_h, s_l=s_l,
                      Lkeep=Lk, idx=idx)
    torch.cuda.synchronize()
    assert torch.equal(s_h.cpu(), g["s_h"]) and torch.equal(s_l.cpu(), g["s_l"])
    assert torch.equal(Lk.cpu(), g["Lkeep"]) and torch.equal(idx.cpu(), g["idx"])
    assert torch.equal(Y.cpu(), g["Y"])
    Yd = tsa.tsa_layer(d["Q"], d["K"], d["V"], d["X"], is_sparse=False).cpu()
    O = tsa.tsa_attn(tsa.dims(d["Q"], d["K"]), d["Q"], d["K"], d["V"], None, dense=True)
    assert torch.equal(Yd, tsa.tsa_scatter_residual(tsa.dims(d["Q"], d["K"]), O, None, None,
                                                    d["X"]).cpu())


@pytest.mark.parametrize("wl,L", [("llama8b_4k", None), ("llama8b_32k", 16384)])
def test_layer_launch_chain_with_and_without_stage_events(wl, L):
    """Without stage events tsa_layer launches the kernels after the scoring as a
    programmatic-dependent chain; with them, each waits for its event.  Both give the same
    layer bit for bit, layer after layer in place (each layer reads the Y the one before
    wrote), also through the grid-wide budget and selection of rows over 8192 tokens."""
    x = make_workload(wl, seed=4, L=L)
    d = _dev(x)
    outs = []
    for use_events in (False, True):
        Y = d["X"].clone()
        Lk = torch.empty(1, dtype=torch.int32, device="cuda")
        idx = torch.empty(1, 32, Y.shape[1], dtype=torch.int32, device="cuda")
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(7)] if use_events else None
        for e in ev or []:
            e.record()  # creates the event (torch makes it on first use)
        for _ in range(3):
            tsa.tsa_layer(d["Q"], d["K"], d["V"], Y, Y, q=16, tau=0.01, Lkeep=Lk, idx=idx,
                          stage_events=ev)
        torch.cuda.synchronize()
        outs.append((Y.cpu(), Lk.cpu(), idx.cpu()))
    for a, b in zip(outs[0], outs[1]):
        assert torch.equal(a, b)


@pytest.mark.parametrize("L", [1, 129, 1000, 4096, 8192])
def test_layer_budget_and_select_in_one_launch_match_the_oracle(L):
    """Rows of up to 8192 tokens take budget and selection in one launch inside tsa_layer
    (every head's CTA recomputes its batch element's budget).  L' and every index list
    equal the oracle's on the GPU's scores, for tau = 0 (keep all), a normal tau, and a
    tau close to 1 (keep few), with two batch elements."""
    x = make_inputs(2, L, 8, 2, 64, torch.bfloat16, seed=L + 5)
    d = _dev(x)
    for tau in (0.0, 0.01, 0.999):
        s_h = torch.empty(2, 8, L, device="cuda")
        s_l = torch.empty(2, L, device="cuda")
        Lk = torch.empty(2, dtype=torch.int32, device="cuda")
        idx = torch.empty(2, 8, L, dtype=torch.int32, device="cuda")
        tsa.tsa_layer(d["Q"], d["K"], d["V"], d["X"], q=16, tau=tau, s_h=s_h, s_l=s_l,
                      Lkeep=Lk, idx=idx)
        lk, _ = oracle.budget(s_l.cpu().numpy(), tau)
        np.testing.assert_array_equal(Lk.cpu().numpy(), lk, err_msg=str(tau))
        np.testing.assert_array_equal(idx.cpu().numpy(), oracle.select(s_h.cpu().numpy(), lk),
                                      err_msg=str(tau))


def test_scores_are_deterministic():
    x = _dev(make_workload("llama8b_4k", seed=3))
    a = tsa.tsa_score(x["Q"], x["K"], 16)
    b = tsa.tsa_score(x["Q"], x["K"], 16)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_headline_128k_sampled():
    """The 128K LLaMA-shaped layer in the benchmark's launch configuration (tsa_layer),
    checked on every score and index and on sampled output rows."""
    L, H, q, tau = 131072, 32, 16, 0.01
    x = make_workload("llama8b_128k", seed=0)
    d = _dev(x)
    s_h = torch.empty(1, H, L, device="cuda")
    s_l = torch.empty(1, L, device="cuda")
    Lk = torch.empty(1, dtype=torch.int32, device="cuda")
    idx = torch.empty(1, H, L, dtype=torch.int32, device="cuda")
    Y = tsa.tsa_layer(d["Q"], d["K"], d["V"], d["X"], q=q, tau=tau, s_h=s_h, s_l=s_l,
                      Lkeep=Lk, idx=idx).cpu()
    s_h, s_l, Lk, idx = s_h.cpu().numpy(), s_l.cpu().numpy(), Lk.cpu().numpy(), idx.cpu().numpy()
    del d
    ref_h, ref_l = oracle.score(x["Q"], x["K"], q)
    assert_scores_close(s_h, ref_h, "s_h@128K")
    assert_scores_close(s_l, ref_l, "s_l@128K")
    lk, _ = oracle.budget(s_l, tau)
    np.testing.assert_array_equal(Lk, lk)
    np.testing.assert_array_equal(idx, oracle.select(s_h, lk))
    rng = np.random.default_rng(0)
    toks = sorted(set(rng.integers(0, L, 6).tolist()) | {0, 3, L - 1})
    Xd = x["X"].double().numpy()
    Yd = Y.double().numpy()
    rows, where = [], []
    for h in range(H):
        pos = {int(t): i for i, t in enumerate(idx[0, h, :lk[0]])}
        for t in toks:
            seg = slice(h * 128, (h + 1) * 128)
            if t in pos:
                rows.append((0, h, pos[t]))
                where.append((t, seg))
            else:
                np.testing.assert_array_equal(Yd[0, t, seg], Xd[0, t, seg])
    vals = oracle.attend_rows(x["Q"], x["K"], x["V"], idx, lk, rows)
    for (t, seg), o in zip(where, vals):
        ref = Xd[0, t, seg] + o
        assert np.all(np.abs(Yd[0, t, seg] - ref) <= 2e-2 + 2.0 ** -8 * np.abs(ref))


def test_attention_is_deterministic():
    """Repeated launches on the same inputs give bit-identical outputs (no races)."""
    x = _dev(make_workload("llama8b_4k", seed=2))
    dm = tsa.dims(x["Q"], x["K"])
    ws = tsa.workspace(dm, 16)
    s_h, s_l = tsa.tsa_score(x["Q"], x["K"], 16, ws=ws)
    Lk = tsa.tsa_budget(dm, s_l, 0.005, ws=ws)
    idx = tsa.tsa_select(dm, s_h, Lk, ws=ws)
    Qh, Kh, Vh = tsa.tsa_gather_qkv(x["Q"], x["K"], x["V"], idx, Lk, ws=ws)
    lk = int(Lk.item())
    ref = tsa.tsa_attn(dm, Qh, Kh, Vh, Lk, ws=ws)[:, :, :lk].clone()
    refd = tsa.tsa_attn(dm, x["Q"], x["K"], x["V"], None, dense=True, ws=ws).clone()
    for _ in range(8):
        assert torch.equal(tsa.tsa_attn(dm, Qh, Kh, Vh, Lk, ws=ws)[:, :, :lk], ref)
        assert torch.equal(tsa.tsa_attn(dm, x["Q"], x["K"], x["V"], None, dense=True, ws=ws), refd)
    assert tsa.tsa_get_device_status(ws) == 0


@pytest.mark.parametrize("H,Hkv,q,L", [(8, 1, 16, 2000),    # 128 query columns per group
                                       (16, 1, 16, 1500),   # 256: query rows on the lanes
                                       (8, 2, 64, 1300),    # q = 64 (the sweep's larger q)
                                       (6, 2, 7, 777),      # odd sizes: 21 columns
                                       (4, 4, 16, 3000)])   # MHA (one head per group)
def test_scoring_shapes(H, Hkv, q, L):
    x = make_inputs(1, L, H, Hkv, 128, torch.bfloat16, seed=H * 100 + q)
    d = _dev(x)
    s_h, s_l = tsa.tsa_score(d["Q"], d["K"], q)
    ref_h, ref_l = oracle.score(x["Q"], x["K"], q)
    assert_scores_close(s_h.cpu().numpy(), ref_h, "s_h")
    assert_scores_close(s_l.cpu().numpy(), ref_l, "s_l")


def test_scoring_many_groups_takes_several_launches():
    """Single-wave kernel (the default): B * Hkv = 160 KV groups exceed one cooperative
    launch (one CTA per SM), so the scoring runs in two launches and the layer score in
    its own kernels.  Both paths equal the oracle; a 2-sample batch (one launch, layer
    score inside the scoring kernel) checks the fused path with B > 1.  (The opt-in
    wave-scheduled kernel covers any number of groups in one launch; its tests are in
    test_gpu_score_wave.py.)"""
    for B, Hkv, L in ((20, 8, 200), (2, 8, 700)):
        x = make_inputs(B, L, Hkv * 2, Hkv, 64, torch.bfloat16, seed=B)
        d = _dev(x)
        s_h, s_l = tsa.tsa_score(d["Q"], d["K"], 16)
        ref_h, ref_l = oracle.score(x["Q"], x["K"], 16)
        assert_scores_close(s_h.cpu().numpy(), ref_h, "s_h B=%d" % B)
        assert_scores_close(s_l.cpu().numpy(), ref_l, "s_l B=%d" % B)


def test_layer_replays_bitwise_in_a_cuda_graph():
    """The whole layer is stream-capturable: a captured replay equals eager calls."""
    x = make_inputs(1, 3000, 32, 8, 128, torch.bfloat16, seed=61)
    d = _dev(x)
    dm = tsa.dims(d["Q"], d["K"])
    ws = tsa.workspace(dm, 16, layer=True)
    Y = torch.empty_like(d["X"])
    run = lambda: tsa.tsa_layer(d["Q"], d["K"], d["V"], d["X"], Y, q=16, tau=0.01, ws=ws)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        run()
    torch.cuda.current_stream().wait_stream(side)
    want = run().clone()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run()
    Y.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert tsa.tsa_get_device_status(ws) == 0
    assert torch.equal(Y, want)
