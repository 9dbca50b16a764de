"""GPU parity of the budget and score variants (fixed-ratio budget, pooled head scores)
against the oracle, through the C ABI.

Tolerances:
  * fixed budget, max pooling, budget and selection on the GPU's scores: bit-exact;
  * mean pooling: the fp32 sum of `width` positive terms in token order and one
    division, against the fp64 mean of the same fp32 inputs: relative (width + 1) * 2^-23;
  * layer scores s_l: relative 1e-5, as for the plain scores;
  * attention and Y: as in test_gpu_parity.
"""
import numpy as np
import pytest
import torch

import oracle
from token_sparse_attention_dtc_b200 import tsa
from token_sparse_attention_dtc_b200.inputs import make_inputs

from test_gpu_parity import ATOL, HALF_ULP, assert_scores_close

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("L", [1, 1000, 131072])
def test_budget_fixed_matches_oracle(L):
    dm = tsa.Dims(3, L, 32, 8, 128, tsa.TSA_BF16)
    for s in (0.0, 0.123, 0.3, 0.5, 0.999, 1.0):
        lk = tsa.tsa_budget_fixed(dm, s)
        np.testing.assert_array_equal(lk.cpu().numpy(), oracle.budget_fixed(3, L, s))


def _gpu_scores(B, L, H, Hkv, seed, q=16):
    x = make_inputs(B, L, H, Hkv, 128, torch.bfloat16, seed=seed)
    Q, K = x["Q"].cuda(), x["K"].cuda()
    s_h, s_l = tsa.tsa_score(Q, K, q)
    return tsa.dims(Q, K), s_h


@pytest.mark.parametrize("L", [5, 2 * 2048 + 1, 5000])
@pytest.mark.parametrize("width", [1, 3, 7, 63, 255])
def test_pool_matches_oracle(L, width):
    dm, s_h = _gpu_scores(2, L, 8, 2, seed=L + width)
    raw = s_h.cpu().numpy()
    for kind in (tsa.POOL_MAX, tsa.POOL_MEAN):
        p, sl = tsa.tsa_pool_scores(dm, s_h, kind, width)
        got = p.cpu().numpy().astype(np.float64)
        ref_p, ref_sl = oracle.pool(raw, kind, width)
        if kind == tsa.POOL_MAX:
            np.testing.assert_array_equal(got, ref_p)
        else:
            rel = np.abs(got - ref_p) / np.maximum(ref_p, 1e-30)
            assert rel.max() <= (width + 1) * 2.0 ** -23, rel.max()
        assert_scores_close(sl.cpu().numpy(), ref_sl, "pooled s_l")


def test_pool_rejects_bad_arguments_before_launch():
    dm, s_h = _gpu_scores(1, 64, 4, 4, seed=3)
    n0 = tsa.kernel_launches()
    for kind, width, code in ((0, 3, 1), (3, 3, 1), (1, 4, 1), (2, 257, 3)):
        with pytest.raises(tsa.TSAError) as e:
            tsa.tsa_pool_scores(dm, s_h, kind, width)
        assert e.value.status == code
    with pytest.raises(tsa.TSAError):
        tsa.tsa_pool_scores(dm, s_h, 1, 3, s_h_out=s_h)   # output overlaps input
    assert tsa.kernel_launches() == n0


def _check_y(x, idx, lk, Y):
    """Y against the oracle's attention on these indices (all heads)."""
    Q, K, V, X = x["Q"], x["K"], x["V"], x["X"]
    dt, dd, H = Q.dtype, Q.shape[3], Q.shape[2]
    Oh = oracle.attend(Q, K, V, idx, lk)
    _, Y_ref = oracle.decompress_residual(Oh, idx, lk, X)
    Yg = Y.double().numpy()
    Xd = X.double().numpy()
    for b in range(Q.shape[0]):
        for h in range(H):
            seg = slice(h * dd, (h + 1) * dd)
            kept, rest = idx[b, h, :lk[b]], idx[b, h, lk[b]:]
            np.testing.assert_array_equal(Yg[b, rest, seg], Xd[b, rest, seg])
            if len(kept):
                diff = np.abs(Yg[b, kept, seg] - Y_ref[b, kept, seg])
                bound = ATOL[dt] + HALF_ULP[dt] * np.abs(Y_ref[b, kept, seg])
                assert np.all(diff <= bound), "Y max excess %.3g" % (diff - bound).max()


@pytest.mark.parametrize("variant", ["pool_max", "pool_mean", "fixed", "fixed_pool"])
def test_layer_ex_matches_oracle(variant):
    B, L, H, Hkv, q, tau = 2, 1000, 8, 2, 16, 0.02
    x = make_inputs(B, L, H, Hkv, 128, torch.bfloat16, seed=41)
    d = {k: v.cuda() for k, v in x.items()}
    pool = {"pool_max": tsa.POOL_MAX, "pool_mean": tsa.POOL_MEAN, "fixed": tsa.POOL_NONE,
            "fixed_pool": tsa.POOL_MAX}[variant]
    sparsity = 0.3 if variant.startswith("fixed") else None
    width = 7 if pool else 1
    s_h = torch.empty(B, H, L, device="cuda")
    s_l = torch.empty(B, L, device="cuda")
    Lk = torch.empty(B, dtype=torch.int32, device="cuda")
    idx = torch.empty(B, H, L, dtype=torch.int32, device="cuda")
    Y = tsa.tsa_layer(d["Q"], d["K"], d["V"], d["X"], q=q, tau=tau, s_h=s_h, s_l=s_l,
                      Lkeep=Lk, idx=idx, sparsity=sparsity, pool=pool, pool_width=width)
    raw, _ = tsa.tsa_score(d["Q"], d["K"], q)
    torch.cuda.synchronize()
    raw = raw.cpu().numpy()
    g_sh, g_sl = s_h.cpu().numpy(), s_l.cpu().numpy()
    # the scores selection used: the pooled GPU scores (pooling checked above), else raw
    if pool:
        ref_p, ref_sl = oracle.pool(raw, pool, width)
        if pool == tsa.POOL_MAX:
            np.testing.assert_array_equal(g_sh.astype(np.float64), ref_p)
        else:
            assert np.max(np.abs(g_sh - ref_p) / np.maximum(ref_p, 1e-30)) <= 8 * 2.0 ** -23
        assert_scores_close(g_sl, ref_sl, "layer s_l")
    else:
        np.testing.assert_array_equal(g_sh, raw)
    lk = (oracle.budget_fixed(B, L, sparsity) if sparsity is not None
          else oracle.budget(g_sl, tau)[0])
    np.testing.assert_array_equal(Lk.cpu().numpy(), lk)
    ref_idx = oracle.select(g_sh, lk)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)
    _check_y(x, ref_idx, lk, Y.cpu())


# ---------------------------------------------------------------- drift pass
def _drift_check(h, eps=1e-6, delta=0.5):
    R, mask = tsa.tsa_drift(h.cuda(), eps=eps, delta=delta)
    R, mask = R.cpu().numpy(), mask.cpu().numpy()
    ref = oracle.drift(h, eps=eps)
    rel = np.abs(R - ref) / np.maximum(np.abs(ref), 1e-30)
    assert rel.max() <= 1e-5, rel.max()
    np.testing.assert_array_equal(mask, oracle.drift_mask(R, delta))   # decision on GPU's R
    return R, mask


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("T", [1, 100, 1000])
def test_drift_matches_oracle(dtype, T):
    g = torch.Generator().manual_seed(T)
    N, D = 6, 256
    steps = torch.rand(N, generator=g) * 0.5                  # a different drift per layer
    h = [torch.randn(T, D, generator=g)]
    for l in range(N):
        h.append(h[-1] + steps[l] * torch.randn(T, D, generator=g))
    _drift_check(torch.stack(h).to(dtype).contiguous(), delta=0.5)


@pytest.mark.parametrize("dtype,N,T,D", [
    (torch.float32, 4, 300, 4096),     # 16 KB rows: four 4 KB slices per token
    (torch.bfloat16, 3, 70, 16384),    # 32 KB rows: eight slices
    (torch.float32, 3, 100, 5120),     # 20 KB rows: five slices
    (torch.bfloat16, 4, 500, 3072),    # 6 KB rows: three 2 KB slices
    (torch.bfloat16, 2, 200, 768),     # 1.5 KB rows: three 512-byte slices
    (torch.bfloat16, 3, 9000, 256),    # more tokens than partial slots (ragged wrap)
    (torch.float32, 5, 4099, 96),      # 384-byte rows: the generic walk, 3 tokens past the slots
])
def test_drift_wide_rows_and_slot_wrap(dtype, N, T, D):
    g = torch.Generator().manual_seed(N * T + D)
    steps = 0.05 + torch.rand(N, generator=g) * 0.5
    h = [torch.randn(T, D, generator=g)]
    for l in range(N):
        h.append(h[-1] + steps[l] * torch.randn(T, D, generator=g))
    _drift_check(torch.stack(h).to(dtype).contiguous(), delta=0.5)


def test_drift_bench_shape_8192_tokens():
    """The bench's bf16 shape at 8192 tokens (two tokens per partial slot), with 4 of its 32
    layers: the walk, the slots and the final sum are those of the timed launches."""
    g = torch.Generator().manual_seed(8192)
    N, T, D = 4, 8192, 4096
    h = [torch.randn(T, D, generator=g)]
    for l in range(N):
        h.append(h[-1] * 0.95 + (0.1 + 0.1 * l) * torch.randn(T, D, generator=g))
    R, mask = _drift_check(torch.stack(h).to(torch.bfloat16).contiguous())
    assert list(mask) == [1, 1, 0, 0]


def test_drift_identical_states_and_determinism():
    h = torch.randn(1, 300, 512).to(torch.bfloat16).expand(9, 300, 512).contiguous()
    R, mask = _drift_check(h)
    assert np.all(R == 0) and list(mask) == [1, 1, 1, 1, 0, 0, 0, 0]
    x = torch.randn(33, 257, 1024, dtype=torch.bfloat16).cuda()
    a = tsa.tsa_drift(x)
    b = tsa.tsa_drift(x)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_drift_llama_width_32_layers():
    g = torch.Generator().manual_seed(5)
    N, T, D = 32, 512, 4096
    h = [torch.randn(T, D, generator=g)]
    for l in range(N):
        h.append(h[-1] * 0.9 + (0.05 + 0.01 * (l % 7)) * torch.randn(T, D, generator=g))
    R, mask = _drift_check(torch.stack(h).to(torch.bfloat16).contiguous())
    assert mask.sum() == 16


# ---------------------------------------------------------------- direct-gather attention
def _staged(d, dm, Lk, idx):
    Qh, Kh, Vh = tsa.tsa_gather_qkv(d["Q"], d["K"], d["V"], idx, Lk)
    Oh = tsa.tsa_attn(dm, Qh, Kh, Vh, Lk)
    return tsa.tsa_scatter_residual(dm, Oh, idx, Lk, d["X"])


@pytest.mark.parametrize("B,L,H,Hkv,hd", [(1, 4096, 32, 8, 128), (2, 1000, 8, 2, 128),
                                           (2, 5000, 8, 8, 128), (2, 1500, 8, 2, 64)])
def test_attn_gather_matches_oracle_and_staged_path(B, L, H, Hkv, hd):
    """The fused compress + attention + decompress against the oracle (its selection
    re-run on the GPU's scores, its attention on those indices), in place and out of
    place, and bit for bit against the staged path."""
    x = make_inputs(B, L, H, Hkv, hd, torch.bfloat16, seed=L + H)
    d = {k: v.cuda() for k, v in x.items()}
    dm = tsa.dims(d["Q"], d["K"])
    s_h, s_l = tsa.tsa_score(d["Q"], d["K"], 16)
    s_h_np = s_h.cpu().numpy()
    for keep in (None, [0] * B, [1] * B, [L] * B, [L // 3 + 7 * b for b in range(B)]):
        Lk = (tsa.tsa_budget(dm, s_l, 0.02) if keep is None
              else torch.tensor(keep, dtype=torch.int32, device="cuda"))
        idx = tsa.tsa_select(dm, s_h, Lk)
        lk = Lk.cpu().numpy()
        ref_idx = oracle.select(s_h_np, lk)
        np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)
        want = _staged(d, dm, Lk, idx)
        ws = tsa.workspace(dm, 1)
        got = tsa.tsa_attn_gather(d["Q"], d["K"], d["V"], idx, Lk, d["X"], ws=ws)
        Yi = d["X"].clone()
        tsa.tsa_attn_gather(d["Q"], d["K"], d["V"], idx, Lk, Yi, Yi, ws=ws)
        assert tsa.tsa_get_device_status(ws) == 0
        _check_y(x, ref_idx, lk, got.cpu())
        _check_y(x, ref_idx, lk, Yi.cpu())
        assert torch.equal(got, want), keep
        assert torch.equal(Yi, want), keep
        if keep is not None and keep[0] == 0:
            assert torch.equal(got, d["X"])


def test_layer_direct_gather_matches_oracle_and_staged_layer():
    x = make_inputs(2, 3000, 32, 8, 128, torch.bfloat16, seed=77)
    d = {k: v.cuda() for k, v in x.items()}
    B, L, H = 2, 3000, 32
    out = {}
    for name, kw in (("tau", dict(tau=0.01)), ("fixed", dict(sparsity=0.5))):
        s_h = torch.empty(B, H, L, device="cuda")
        s_l = torch.empty(B, L, device="cuda")
        Lk = torch.empty(B, dtype=torch.int32, device="cuda")
        Y2 = tsa.tsa_layer(d["Q"], d["K"], d["V"], d["X"], q=16, direct=True, s_h=s_h, s_l=s_l,
                           Lkeep=Lk, **kw)
        Y1 = tsa.tsa_layer(d["Q"], d["K"], d["V"], d["X"], q=16, **kw)
        assert torch.equal(Y1, Y2), name
        g_sh, g_sl = s_h.cpu().numpy(), s_l.cpu().numpy()
        ref_h, ref_l = oracle.score(x["Q"], x["K"], 16)
        assert_scores_close(g_sh, ref_h, "s_h")
        assert_scores_close(g_sl, ref_l, "s_l")
        lk = (oracle.budget(g_sl, 0.01)[0] if name == "tau"
              else oracle.budget_fixed(B, L, 0.5))
        np.testing.assert_array_equal(Lk.cpu().numpy(), lk)
        _check_y(x, oracle.select(g_sh, lk), lk, Y2.cpu())
        out[name] = Y2
    # in place: Y == X, the unselected segments untouched
    Yi = d["X"].clone()
    tsa.tsa_layer(d["Q"], d["K"], d["V"], Yi, Yi, q=16, tau=0.01, direct=True)
    assert torch.equal(Yi, out["tau"])


def test_attn_gather_reports_a_bad_index():
    x = make_inputs(1, 512, 4, 4, 128, torch.bfloat16, seed=5)
    d = {k: v.cuda() for k, v in x.items()}
    dm = tsa.dims(d["Q"], d["K"])
    idx = torch.arange(512, dtype=torch.int32, device="cuda").repeat(1, 4, 1).contiguous()
    idx[0, 2, 10] = 512                      # out of range: skipped and reported
    Lk = torch.tensor([512], dtype=torch.int32, device="cuda")
    ws = tsa.workspace(dm, 1)
    tsa.tsa_attn_gather(d["Q"], d["K"], d["V"], idx, Lk, d["X"], ws=ws)
    assert tsa.tsa_get_device_status(ws) == 1            # TSA_ERR_INVALID_ARG


# ---------------------------------------------------------------- block-sparse attention
def _keep_to_words(keep):
    B, H, NP, NB = keep.shape
    NW = (NB + 31) // 32
    w = np.zeros((B, H, NP, NW), np.uint32)
    for j in range(NB):
        w[..., j // 32] |= (keep[..., j].astype(np.uint32) << np.uint32(j % 32))
    return w


def _compressed(B, L, H, Hkv, seed, keep):
    x = make_inputs(B, L, H, Hkv, 128, torch.bfloat16, seed=seed)
    d = {k: v.cuda() for k, v in x.items()}
    dm = tsa.dims(d["Q"], d["K"])
    s_h, _ = tsa.tsa_score(d["Q"], d["K"], 16)
    Lk = torch.tensor(keep, dtype=torch.int32, device="cuda")
    idx = tsa.tsa_select(dm, s_h, Lk)
    Qh, Kh, Vh = tsa.tsa_gather_qkv(d["Q"], d["K"], d["V"], idx, Lk)
    return x, d, dm, Lk, idx, Qh, Kh, Vh


@pytest.mark.parametrize("B,L,H,Hkv,keep,theta", [(1, 4096, 8, 2, [4096], 1.0),
                                                  (2, 3000, 4, 4, [3000, 1111], 0.5),
                                                  (1, 2600, 8, 2, [2555], 0.0)])
def test_block_select_and_attention_match_oracle(B, L, H, Hkv, keep, theta):
    x, d, dm, Lk, idx, Qh, Kh, Vh = _compressed(B, L, H, Hkv, seed=L + H, keep=keep)
    z, mask = tsa.tsa_block_select(dm, Qh, Kh, Lk, theta)
    zg = z.cpu().numpy()
    ref = oracle.block_logits(x["Q"], x["K"], idx.cpu().numpy(), keep)
    fin = np.isfinite(ref)
    assert np.array_equal(fin, np.isfinite(zg))
    assert np.max(np.abs(zg[fin] - ref[fin])) <= 1e-4 * max(1.0, np.max(np.abs(ref[fin])))
    want = _keep_to_words(oracle.block_select(zg, np.array(keep, np.int32), theta))
    np.testing.assert_array_equal(mask.cpu().numpy().view(np.uint32), want)
    Oh = tsa.tsa_attn_block(dm, Qh, Kh, Vh, Lk, mask)
    keep_u8 = oracle.block_select(zg, np.array(keep, np.int32), theta)
    rng = np.random.default_rng(0)
    rows = [(b, h, int(i)) for b in range(B) for h in (0, H - 1)
            for i in np.unique(np.concatenate([[0, 127, 128, 255, 256, keep[b] - 1],
                                                 rng.integers(0, keep[b], 12)]))]
    got = Oh.cpu().double().numpy()[tuple(np.asarray(rows).T)]
    ref_o = oracle.attend_block_rows(x["Q"], x["K"], x["V"], idx.cpu().numpy(), keep, keep_u8, rows)
    assert np.max(np.abs(got - ref_o)) <= 2e-2
    if theta == 0.0:
        assert keep_u8.sum() < sum(2 * ((k + 255) // 256) ** 2 for k in keep) * H  # sparse


def test_block_theta_huge_equals_full_compressed_attention():
    x, d, dm, Lk, idx, Qh, Kh, Vh = _compressed(1, 5000, 8, 2, seed=9, keep=[4800])
    _, mask = tsa.tsa_block_select(dm, Qh, Kh, Lk, 3e38, logits=False)
    got = tsa.tsa_attn_block(dm, Qh, Kh, Vh, Lk, mask)
    want = tsa.tsa_attn(dm, Qh, Kh, Vh, Lk)
    assert torch.equal(got[:, :, :4800], want[:, :, :4800])   # rows >= L' are not written


def test_layer_block_theta_equals_manual_chain():
    x = make_inputs(1, 4096, 32, 8, 128, torch.bfloat16, seed=12)
    d = {k: v.cuda() for k, v in x.items()}
    dm = tsa.dims(d["Q"], d["K"])
    Lk = torch.empty(1, dtype=torch.int32, device="cuda")
    idx = torch.empty(1, 32, 4096, dtype=torch.int32, device="cuda")
    Y = tsa.tsa_layer(d["Q"], d["K"], d["V"], d["X"], q=16, tau=0.01, Lkeep=Lk, idx=idx,
                      block_theta=0.5)
    Qh, Kh, Vh = tsa.tsa_gather_qkv(d["Q"], d["K"], d["V"], idx, Lk)
    _, mask = tsa.tsa_block_select(dm, Qh, Kh, Lk, 0.5)
    Oh = tsa.tsa_attn_block(dm, Qh, Kh, Vh, Lk, mask)
    assert torch.equal(Y, tsa.tsa_scatter_residual(dm, Oh, idx, Lk, d["X"]))


@pytest.mark.parametrize("d", [64, 128])
def test_block_select_fp32_matches_oracle(d):
    B, L, H, Hkv, keep, theta = 1, 1500, 4, 2, [1400], 0.3
    x = make_inputs(B, L, H, Hkv, d, torch.float32, seed=d)
    dd = {k: v.cuda() for k, v in x.items()}
    dm = tsa.dims(dd["Q"], dd["K"])
    s_h, _ = tsa.tsa_score(dd["Q"], dd["K"], 16)
    Lk = torch.tensor(keep, dtype=torch.int32, device="cuda")
    idx = tsa.tsa_select(dm, s_h, Lk)
    Qh, Kh, _ = tsa.tsa_gather_qkv(dd["Q"], dd["K"], dd["V"], idx, Lk)
    z, mask = tsa.tsa_block_select(dm, Qh, Kh, Lk, theta)
    zg = z.cpu().numpy()
    ref = oracle.block_logits(x["Q"], x["K"], idx.cpu().numpy(), keep)
    fin = np.isfinite(ref)
    assert np.array_equal(fin, np.isfinite(zg))
    assert np.max(np.abs(zg[fin] - ref[fin])) <= 1e-5 * max(1.0, np.max(np.abs(ref[fin])))
    want = _keep_to_words(oracle.block_select(zg, np.array(keep, np.int32), theta))
    np.testing.assert_array_equal(mask.cpu().numpy().view(np.uint32), want)
