"""Pins for the CPU oracle (no GPU).

Each test ties an oracle function to something other than itself: a library
routine (torch float64 scaled_dot_product_attention / softmax), a closed form,
or brute-force enumeration on tiny inputs.  Together they are chosen so that a
dropped term, a wrong sign, index or head mapping, or a transposed operand in
the oracle fails at least one of them.
"""
import itertools
from fractions import Fraction

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from token_sparse_attention_dtc_b200.inputs import make_inputs


def _rand(B, L, H, Hkv, d, dtype=torch.float32, seed=0):
    return make_inputs(B, L, H, Hkv, d, dtype, seed=seed, shift=2.0, heavy_frac=0.1)


def _sdpa_weights_last_rows(Q, K, q):
    """Causal softmax weights of the last q query rows, via SDPA with V = I.

    Returns A [B, H, q_eff, L] in float64.
    """
    B, L, H, d = Q.shape
    Hkv = K.shape[2]
    qe = min(q, L)
    Qd = Q.double().permute(0, 2, 1, 3)[:, :, L - qe:]          # [B,H,qe,d]
    Kd = K.double().permute(0, 2, 1, 3).repeat_interleave(H // Hkv, dim=1)  # [B,H,L,d]
    eye = torch.eye(L, dtype=torch.float64).expand(B, H, L, L)
    pos = torch.arange(L - qe, L).view(qe, 1)
    mask = torch.arange(L).view(1, L) <= pos                     # [qe, L]
    return F.scaled_dot_product_attention(Qd, Kd, eye, attn_mask=mask)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("B,L,H,Hkv,d,q", [(2, 37, 4, 2, 16, 5), (1, 9, 2, 1, 8, 16),
                                           (1, 64, 8, 2, 32, 16)])
def test_score_matches_sdpa_weights(dtype, B, L, H, Hkv, d, q):
    x = _rand(B, L, H, Hkv, d, dtype, seed=L)
    s_h, s_l = oracle.score(x["Q"], x["K"], q)
    A = _sdpa_weights_last_rows(x["Q"], x["K"], q)
    ref_sh = A.sum(dim=2).numpy()
    np.testing.assert_allclose(s_h, ref_sh, rtol=1e-11, atol=1e-14)
    u = ref_sh.sum(axis=1)
    np.testing.assert_allclose(s_l, u / u.sum(axis=1, keepdims=True), rtol=1e-11, atol=1e-15)


def test_score_single_query_is_softmax():
    x = _rand(1, 50, 1, 1, 16, seed=3)
    s_h, s_l = oracle.score(x["Q"], x["K"], 1)
    z = (x["K"][0, :, 0].double() @ x["Q"][0, -1, 0].double()) / 4.0
    ref = torch.softmax(z, dim=0).numpy()
    np.testing.assert_allclose(s_h[0, 0], ref, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(s_l[0], ref, rtol=1e-12, atol=1e-15)


def test_score_identical_keys_closed_form():
    B, L, H, Hkv, d, q = 1, 40, 4, 2, 8, 7
    x = _rand(B, L, H, Hkv, d, seed=5)
    K = x["K"].clone()
    K[:] = K[:, :1]  # every key equals key 0 of its head
    s_h, _ = oracle.score(x["Q"], K, q)
    p = np.arange(L - q, L)
    ref = np.array([np.sum(1.0 / (p[p >= t] + 1)) for t in range(L)])
    for h in range(H):
        np.testing.assert_allclose(s_h[0, h], ref, rtol=1e-12)


@pytest.mark.parametrize("q", [1, 16, 100])
def test_score_mass_invariants(q):
    B, L, H, Hkv, d = 2, 33, 4, 4, 16
    x = _rand(B, L, H, Hkv, d, seed=11)
    s_h, s_l = oracle.score(x["Q"], x["K"], q)
    np.testing.assert_allclose(s_h.sum(axis=2), min(q, L), rtol=1e-12)
    np.testing.assert_allclose(s_l.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    # the last query only is the last one to see the last key
    assert np.all(s_h >= 0)


def test_score_gqa_head_mapping():
    """Query head h must read KV head h // (H/Hkv): change one KV head only."""
    B, L, H, Hkv, d = 1, 20, 4, 2, 8
    x = _rand(B, L, H, Hkv, d, seed=2)
    a, _ = oracle.score(x["Q"], x["K"], 4)
    K2 = x["K"].clone()
    K2[:, :, 1] = torch.randn(B, L, d, generator=torch.Generator().manual_seed(9))
    b, _ = oracle.score(x["Q"], K2, 4)
    np.testing.assert_array_equal(a[0, :2], b[0, :2])
    assert np.abs(a[0, 2:] - b[0, 2:]).max() > 1e-3


# ---------------------------------------------------------------- budget ---

def _brute_budget(vals, tau):
    """min k such that the k smallest masses (by enumeration) sum to >= tau."""
    L = len(vals)
    fr = [Fraction(float(v)) for v in vals]
    t = Fraction(tau)
    for k in range(0, L + 1):
        best = min(sum(c, Fraction(0)) for c in itertools.combinations(fr, k)) if k else 0
        if best >= t:
            return k
    return L


def test_budget_tau_zero_keeps_all():
    s = np.random.default_rng(0).random((3, 17)).astype(np.float32)
    s /= s.sum(axis=1, keepdims=True)
    lk, _ = oracle.budget(s.astype(np.float32), 0.0)
    assert list(lk) == [17, 17, 17]


@pytest.mark.parametrize("n", [3, 7, 10, 17])
@pytest.mark.parametrize("tau", [0.001, 0.005, 0.01, 0.02, 0.3, 0.75])
def test_budget_uniform_closed_form(n, tau):
    L = 2 ** n
    s = np.full((1, L), 1.0 / L, np.float32)
    lk, dis = oracle.budget(s, tau)
    assert lk[0] == L - int(np.ceil(tau * L))
    assert dis == 0


def test_budget_exact_hit_counts_equality():
    # masses 1/16, 1/16, 1/8, 1/4, 1/2: cumulative 1/16, 1/8, 1/4, 1/2, 1
    s = np.array([[0.25, 0.0625, 0.5, 0.125, 0.0625]], np.float32)
    assert oracle.budget(s, 0.125)[0][0] == 5 - 2
    assert oracle.budget(s, 0.1250001)[0][0] == 5 - 3
    assert oracle.budget(s, 0.0625)[0][0] == 5 - 1
    assert oracle.budget(s, 0.999)[0][0] == 0


@pytest.mark.parametrize("seed", range(12))
def test_budget_bruteforce(seed):
    rng = np.random.default_rng(seed)
    L = int(rng.integers(1, 11))
    v = rng.random(L) ** 3
    v = (v / v.sum()).astype(np.float32)
    for tau in (0.0, 0.01, 0.05, 0.2, 0.5):
        lk, _ = oracle.budget(v[None], tau)
        assert lk[0] == L - _brute_budget(v, tau), (seed, tau)


def test_budget_never_reached_keeps_none():
    s = np.zeros((1, 8), np.float32)
    assert oracle.budget(s, 0.5)[0][0] == 0


# ---------------------------------------------------------------- select ---

def _brute_select(vals, k):
    """Subset of size k with the largest exact sum; ties -> smallest sorted tuple."""
    L = len(vals)
    fr = [Fraction(float(v)) for v in vals]
    best = None
    for c in itertools.combinations(range(L), k):
        key = (sum((fr[i] for i in c), Fraction(0)), tuple(-i for i in c))
        if best is None or key > best[0]:
            best = (key, c)
    return list(best[1]) if best else []


@pytest.mark.parametrize("seed", range(10))
def test_select_bruteforce_with_ties(seed):
    rng = np.random.default_rng(100 + seed)
    L = int(rng.integers(1, 10))
    H = 3
    s = rng.integers(0, 4, size=(1, H, L)).astype(np.float32) / 4  # many ties
    for Lk in range(0, L + 1):
        idx = oracle.select(s, np.array([Lk], np.int32))
        for h in range(H):
            want = _brute_select(s[0, h], Lk)
            assert list(idx[0, h, :Lk]) == want
            rest = sorted(set(range(L)) - set(want))
            assert list(idx[0, h, Lk:]) == rest


def test_select_all_equal_takes_prefix():
    s = np.full((2, 2, 50), 0.25, np.float32)
    idx = oracle.select(s, np.array([13, 50], np.int32))
    assert list(idx[0, 0]) == list(range(50))
    assert list(idx[1, 1]) == list(range(50))


def test_select_strict_order_then_ties():
    s = np.array([[[0.1, 0.5, 0.3, 0.5, 0.2, 0.3]]], np.float32)
    idx = oracle.select(s, np.array([3], np.int32))
    assert list(idx[0, 0]) == [1, 2, 3, 0, 4, 5]


# ---------------------------------------------------------------- attend ---

def _sdpa_dense(Q, K, V):
    B, L, H, d = Q.shape
    G = H // K.shape[2]
    q = Q.double().permute(0, 2, 1, 3)
    k = K.double().permute(0, 2, 1, 3).repeat_interleave(G, dim=1)
    v = V.double().permute(0, 2, 1, 3).repeat_interleave(G, dim=1)
    return F.scaled_dot_product_attention(q, k, v, is_causal=True)  # [B,H,L,d]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_attend_dense_matches_sdpa(dtype):
    x = _rand(2, 23, 4, 2, 16, dtype, seed=4)
    Oh = oracle.attend(x["Q"], x["K"], x["V"], None, None)
    np.testing.assert_allclose(Oh, _sdpa_dense(x["Q"], x["K"], x["V"]).numpy(),
                               rtol=1e-11, atol=1e-13)


def test_attend_compressed_matches_sdpa_on_gathered_rows():
    B, L, H, Hkv, d = 1, 30, 4, 2, 16
    x = _rand(B, L, H, Hkv, d, seed=8)
    rng = np.random.default_rng(1)
    Lk = 11
    idx = np.zeros((B, H, L), np.int32)
    for h in range(H):
        sel = np.sort(rng.choice(L, Lk, replace=False))
        idx[0, h] = np.concatenate([sel, np.setdiff1d(np.arange(L), sel)])
    Oh = oracle.attend(x["Q"], x["K"], x["V"], idx, np.array([Lk], np.int32))
    G = H // Hkv
    for h in range(H):
        S = torch.from_numpy(idx[0, h, :Lk]).long()
        q = x["Q"][0, S, h].double()[None, None]
        k = x["K"][0, S, h // G].double()[None, None]
        v = x["V"][0, S, h // G].double()[None, None]
        ref = F.scaled_dot_product_attention(q, k, v, is_causal=True)[0, 0].numpy()
        np.testing.assert_allclose(Oh[0, h, :Lk], ref, rtol=1e-11, atol=1e-13)
        assert np.all(Oh[0, h, Lk:] == 0)


def test_attend_identical_keys_is_running_mean():
    x = _rand(1, 12, 2, 1, 8, seed=6)
    K = x["K"].clone()
    K[:] = K[:, :1]
    Oh = oracle.attend(x["Q"], K, x["V"], None, None)
    V = x["V"][0, :, 0].double().numpy()
    ref = np.cumsum(V, axis=0) / np.arange(1, 13)[:, None]
    for h in range(2):
        np.testing.assert_allclose(Oh[0, h], ref, rtol=1e-12, atol=1e-14)


def test_attend_single_kept_row_returns_its_value():
    x = _rand(1, 10, 2, 2, 8, seed=7)
    idx = np.tile(np.arange(10, dtype=np.int32), (1, 2, 1))
    idx[0, 1] = np.array([6, 0, 1, 2, 3, 4, 5, 7, 8, 9])
    Oh = oracle.attend(x["Q"], x["K"], x["V"], idx, np.array([1], np.int32))
    np.testing.assert_array_equal(Oh[0, 0, 0], x["V"][0, 0, 0].double().numpy())
    np.testing.assert_array_equal(Oh[0, 1, 0], x["V"][0, 6, 1].double().numpy())


def test_attend_is_linear_in_v():
    x = _rand(1, 16, 2, 1, 8, seed=12)
    a = oracle.attend(x["Q"], x["K"], x["V"], None, None)
    b = oracle.attend(x["Q"], x["K"], x["V"] * 4, None, None)
    np.testing.assert_array_equal(b, 4 * a)


# ------------------------------------------------------- decompress + layer ---

def test_decompress_zero_rows_and_residual():
    B, L, H, Hkv, d = 1, 20, 2, 1, 4
    x = _rand(B, L, H, Hkv, d, seed=13)
    s_h, s_l = oracle.score(x["Q"], x["K"], 4)
    lk, _ = oracle.budget(s_l.astype(np.float32), 0.3)
    assert 0 < lk[0] < L
    idx = oracle.select(s_h.astype(np.float32), lk)
    Oh = oracle.attend(x["Q"], x["K"], x["V"], idx, lk)
    O, Y = oracle.decompress_residual(Oh, idx, lk, x["X"])
    X = x["X"].double().numpy()
    for h in range(H):
        kept = set(idx[0, h, :lk[0]].tolist())
        for t in range(L):
            seg = slice(h * d, (h + 1) * d)
            if t in kept:
                i = list(idx[0, h, :lk[0]]).index(t)
                np.testing.assert_array_equal(O[0, t, seg], Oh[0, h, i])
            else:
                assert np.all(O[0, t, seg] == 0)
                np.testing.assert_array_equal(Y[0, t, seg], X[0, t, seg])
    np.testing.assert_array_equal(Y, X + O)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_layer_tau_zero_equals_dense_attention(dtype):
    x = _rand(1, 25, 4, 2, 16, dtype, seed=21)
    sp = oracle.layer(x["Q"], x["K"], x["V"], x["X"], q=4, tau=0.0)
    de = oracle.layer(x["Q"], x["K"], x["V"], x["X"], q=4, tau=0.0, is_sparse=False)
    assert sp["Lkeep"][0] == 25
    np.testing.assert_allclose(sp["Y"], de["Y"], rtol=0, atol=1e-13)
    ref = _sdpa_dense(x["Q"], x["K"], x["V"]).permute(0, 2, 1, 3).reshape(1, 25, 64)
    np.testing.assert_allclose(de["Y"], x["X"].double().numpy() + ref.numpy(), atol=1e-12)


def test_bf16_decode_matches_torch():
    v = torch.randn(1000).to(torch.bfloat16)
    x = dict(Q=v.view(1, 1000, 1, 1), K=v.view(1, 1000, 1, 1))
    s_h, _ = oracle.score(x["Q"], x["K"], 1, scale=0.0)
    np.testing.assert_allclose(s_h[0, 0], 1.0 / 1000, rtol=1e-14)
    O, Y = oracle.decompress_residual(np.zeros((1, 1, 1000, 1)), None, None,
                                      v.view(1, 1000, 1))
    np.testing.assert_array_equal(Y[0, :, 0], v.double().numpy())


# ---------------------------------------------------------------- budget / score variants
@pytest.mark.parametrize("L", [10, 1000, 131070])
def test_budget_fixed_prunes_the_stated_decimal_fraction(L):
    # The pages' ablation prunes a fixed 30% / 50%: s = m/10 removes exactly m*L/10 tokens.
    for m in range(11):
        lk = oracle.budget_fixed(2, L, m / 10)
        assert list(lk) == [L - m * L // 10] * 2


def test_budget_fixed_limits_and_rejects():
    assert oracle.budget_fixed(1, 7, 0.0)[0] == 7
    assert oracle.budget_fixed(1, 7, 1.0)[0] == 0
    assert oracle.budget_fixed(1, 7, 0.5)[0] == 4          # floor(3.5) pruned
    for bad in (-0.1, 1.5, float("nan")):
        with pytest.raises(ValueError):
            oracle.budget_fixed(1, 7, bad)


def _pool_brute(s, kind, width):
    """Pure-Python restatement on small inputs: clipped windows, index-order sums."""
    r = width // 2
    B, H, L = s.shape
    out = np.zeros_like(s, dtype=np.float64)
    for b in range(B):
        for h in range(H):
            for t in range(L):
                w = [float(s[b, h, u]) for u in range(max(0, t - r), min(L, t + r + 1))]
                out[b, h, t] = max(w) if kind == oracle.POOL_MAX else sum(w) / len(w)
    return out


@pytest.mark.parametrize("kind", [1, 2])
def test_pool_width_one_is_identity(kind):
    s = np.random.default_rng(0).random((2, 3, 17))
    p, sl = oracle.pool(s, kind, 1)
    np.testing.assert_array_equal(p, s)
    np.testing.assert_allclose(sl, s.sum(1) / s.sum(1).sum(1, keepdims=True), rtol=1e-15)


def test_pool_delta_gives_the_clipped_window():
    L, w = 12, 5
    for pos in (0, 1, 6, 11):
        s = np.zeros((1, 1, L))
        s[0, 0, pos] = 1.0
        mx, _ = oracle.pool(s, oracle.POOL_MAX, w)
        mean, _ = oracle.pool(s, oracle.POOL_MEAN, w)
        for t in range(L):
            inside = abs(t - pos) <= 2
            cnt = min(L - 1, t + 2) - max(0, t - 2) + 1
            assert mx[0, 0, t] == (1.0 if inside else 0.0)
            assert mean[0, 0, t] == pytest.approx(1.0 / cnt if inside else 0.0, abs=0, rel=1e-15)


def test_pool_mean_keeps_a_constant_at_the_edges():
    s = np.full((1, 2, 9), 0.125)
    p, sl = oracle.pool(s, oracle.POOL_MEAN, 7)
    np.testing.assert_array_equal(p, s)          # 0.125 * n / n is exact
    np.testing.assert_allclose(sl, 1.0 / 9, rtol=1e-15)


@pytest.mark.parametrize("kind,width", [(1, 3), (1, 7), (2, 3), (2, 9)])
def test_pool_matches_brute_force(kind, width):
    s = np.random.default_rng(width + kind).random((2, 3, 23)).astype(np.float32)
    p, sl = oracle.pool(s, kind, width)
    np.testing.assert_allclose(p, _pool_brute(s, kind, width), rtol=1e-15, atol=0)
    u = p.sum(1)
    np.testing.assert_allclose(sl, u / u.sum(1, keepdims=True), rtol=1e-14)
    np.testing.assert_allclose(sl.sum(1), 1.0, rtol=1e-14)


def test_pool_mean_matches_prefix_sums_and_max_bounds():
    s = np.random.default_rng(5).random((1, 1, 200))
    r = 15
    p, _ = oracle.pool(s, oracle.POOL_MEAN, 2 * r + 1)
    c = np.concatenate([[0.0], np.cumsum(s[0, 0])])
    lo = np.maximum(np.arange(200) - r, 0)
    hi = np.minimum(np.arange(200) + r, 199)
    np.testing.assert_allclose(p[0, 0], (c[hi + 1] - c[lo]) / (hi - lo + 1), rtol=1e-12)
    mx, _ = oracle.pool(s, oracle.POOL_MAX, 2 * r + 1)
    assert np.all(mx >= s) and np.all(mx >= p)


def test_pool_rejects_bad_arguments():
    s = np.ones((1, 1, 4))
    for kind, width in ((3, 3), (1, 2), (2, 0)):
        with pytest.raises(ValueError):
            oracle.pool(s, kind, width)


# ---------------------------------------------------------------- drift pass
def test_drift_identical_states_are_zero_and_mask_takes_lowest_indices():
    h = np.tile(np.random.default_rng(0).standard_normal((1, 6, 16)).astype(np.float32), (9, 1, 1))
    R = oracle.drift(h)
    np.testing.assert_array_equal(R, 0.0)
    np.testing.assert_array_equal(oracle.drift_mask(R, 0.5), [1, 1, 1, 1, 0, 0, 0, 0])


def test_drift_of_scaled_states_is_the_scale_step():
    rng = np.random.default_rng(1)
    c = [2.0, 0.5, 4.0, 1.0, 0.25]
    h = [rng.standard_normal((7, 32)).astype(np.float32)]
    for k in c:
        h.append((h[-1] * np.float32(k)).astype(np.float32))   # exact: powers of two
    R = oracle.drift(np.stack(h), eps=0.0)
    np.testing.assert_allclose(R, [abs(k - 1) for k in c], rtol=1e-12)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_drift_matches_numpy_norms(dtype):
    h = torch.randn(5, 11, 64).to(dtype)
    eps = 1e-3
    R = oracle.drift(h, eps=eps)
    hd = h.double().numpy()
    want = [np.mean(np.linalg.norm(hd[l + 1] - hd[l], axis=1) / (np.linalg.norm(hd[l], axis=1) + eps))
            for l in range(4)]
    np.testing.assert_allclose(R, want, rtol=1e-12)


@pytest.mark.parametrize("N,delta", [(32, 0.5), (5, 0.5), (7, 0.3), (4, 1.0), (4, 0.0)])
def test_drift_mask_brute_force(N, delta):
    rng = np.random.default_rng(N)
    R = rng.integers(0, 4, N).astype(np.float64) / 4        # ties on purpose
    order = sorted(range(N), key=lambda l: (R[l], l))
    want = np.zeros(N, np.int32)
    for rank, l in enumerate(order, start=1):
        want[l] = Fraction(rank, N) <= Fraction(delta)
    np.testing.assert_array_equal(oracle.drift_mask(R, delta), want)
    if N == 32 and delta == 0.5:
        assert want.sum() == 16                               # half the layers sparse


def test_drift_rejects_bad_arguments():
    with pytest.raises(ValueError):
        oracle.drift(np.zeros((1, 3, 4), np.float32))         # needs two states
    with pytest.raises(ValueError):
        oracle.drift_mask(np.zeros(3), 1.5)


# ---------------------------------------------------------------- block-sparse pattern
def _block_case(L=700, H=2, Hkv=1, d=16, seed=0, keep=None):
    x = make_inputs(1, L, H, Hkv, d, torch.float32, seed=seed)
    lk = np.array([L if keep is None else keep], np.int32)
    rng = np.random.default_rng(seed)
    idx = np.stack([np.concatenate([np.sort(p[:lk[0]]), np.sort(p[lk[0]:])])
                    for p in (rng.permutation(L) for _ in range(H))])[None].astype(np.int32)
    return x, idx, lk


def test_block_logits_brute_force():
    x, idx, lk = _block_case(L=600, keep=530)
    z = oracle.block_logits(x["Q"], x["K"], idx, lk, scale=0.25)
    Q, K = x["Q"].double().numpy(), x["K"].double().numpy()
    NP, NB = z.shape[2:]
    assert (NP, NB) == (3, 5)
    for h in range(2):
        S = idx[0, h]
        for p in range(NP):
            rows = range(256 * p, min(256 * p + 256, lk[0]))
            if not len(rows):
                assert np.all(np.isnan(z[0, h, p]))
                continue
            qb = np.mean([Q[0, S[i], h] for i in rows], axis=0)
            for j in range(NB):
                if j >= 2 * p:
                    assert np.isnan(z[0, h, p, j])
                    continue
                kb = np.mean([K[0, S[i], 0] for i in range(128 * j, 128 * j + 128)], axis=0)
                assert z[0, h, p, j] == pytest.approx(0.25 * qb @ kb, rel=1e-12, abs=1e-15)


def test_block_select_rule_and_ties():
    B, H, L = 1, 1, 1024                     # NP = 4, NB = 8
    z = np.full((B, H, 4, 8), np.nan, np.float32)
    z[0, 0, 3, :6] = [0.0, 5.0, 1.0, 4.0, 5.0, 2.0]      # max 5 (twice)
    z[0, 0, 2, :4] = [3.0, 1.0, -1.0, 2.0]
    z[0, 0, 1, :2] = [7.0, 0.0]
    keep = oracle.block_select(z, np.array([L], np.int32), theta=1.0)
    assert list(keep[0, 0, 3]) == [1, 1, 0, 1, 1, 0, 1, 1]   # 0, ties at 5, 4 >= 4, diag 6, 7
    assert list(keep[0, 0, 2]) == [1, 0, 0, 1, 1, 1, 0, 0]   # 0, 2 >= 2, diag 4, 5
    assert list(keep[0, 0, 1]) == [1, 0, 1, 1, 0, 0, 0, 0]   # 0, z1 = 0 < 6, diag 2, 3
    assert list(keep[0, 0, 0]) == [1, 1, 0, 0, 0, 0, 0, 0]   # diag 0, 1
    every = oracle.block_select(z, np.array([L], np.int32), theta=np.inf)
    assert every[0, 0, 3, :8].sum() == 8
    short = oracle.block_select(z, np.array([890], np.int32), theta=0.0)   # pair 3: no block 7
    assert list(short[0, 0, 3]) == [1, 1, 0, 0, 1, 0, 1, 0]


def test_block_attention_with_every_block_is_compressed_attention():
    x, idx, lk = _block_case(L=700, keep=650, seed=3)
    z = oracle.block_logits(x["Q"], x["K"], idx, lk)
    keep = oracle.block_select(z.astype(np.float32), lk, theta=np.inf)
    rows = [(0, h, i) for h in range(2) for i in (0, 1, 127, 128, 255, 256, 300, 511, 512, 649)]
    got = oracle.attend_block_rows(x["Q"], x["K"], x["V"], idx, lk, keep, rows)
    want = oracle.attend_rows(x["Q"], x["K"], x["V"], idx, lk, rows)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-14)


def test_block_attention_matches_masked_softmax():
    x, idx, lk = _block_case(L=640, keep=640, seed=4)
    z = oracle.block_logits(x["Q"], x["K"], idx, lk)
    keep = oracle.block_select(z.astype(np.float32), lk, theta=0.05)
    assert keep.sum() < np.isfinite(z).sum() + 3 * 2 * 3      # something was dropped
    Q, K, V = (x[k].double() for k in ("Q", "K", "V"))
    for h in range(2):
        S = torch.from_numpy(idx[0, h]).long()
        q, k, v = Q[0, S, h], K[0, S, 0], V[0, S, 0]
        logits = (q @ k.T) / np.sqrt(16)
        allowed = torch.zeros(640, 640, dtype=torch.bool)
        for i in range(640):
            blocks = torch.from_numpy(keep[0, h, i // 256].astype(bool))
            allowed[i, : i + 1] = blocks[torch.arange(i + 1) // 128]
        ref = torch.softmax(logits.masked_fill(~allowed, float("-inf")), dim=1) @ v
        rows = [(0, h, i) for i in range(0, 640, 7)]
        got = oracle.attend_block_rows(x["Q"], x["K"], x["V"], idx, lk, keep, rows)
        np.testing.assert_allclose(got, ref[::7].numpy(), rtol=0, atol=1e-13)


def test_oracle_matches_its_stored_regression():
    """The oracle reproduces, bit for bit, the results it stored for one small seeded layer
    (tests/golden/make_oracle_regression.py).  This pins the oracle against unintended
    changes of its arithmetic; the pins above pin it against the pages and mathematics."""
    import importlib.util
    import json
    import os

    here = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
    spec = importlib.util.spec_from_file_location(
        "make_oracle_regression", os.path.join(here, "make_oracle_regression.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    with open(os.path.join(here, "oracle_regression.json")) as f:
        want = json.load(f)
    got = json.loads(json.dumps(mod.compute()))
    for k in ("case", "Lkeep", "idx", "s_l", "s_h", "Oh", "Y"):
        assert got[k] == want[k], k
