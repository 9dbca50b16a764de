"""C-ABI boundary checks that need no GPU.

The library must load, export every entry point include/tsa.h declares, size
workspaces on the host, and reject bad arguments before touching the device.
None of these tests makes a CUDA call that launches work: every call below
fails host-side validation (or is a pure host query).
"""
import ctypes
import os
import re

import pytest

from token_sparse_attention_dtc_b200 import tsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "tsa.h")).read()
    return sorted(set(re.findall(r"TSA_API[^;(]*?\b(tsa_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("tsa_score", "tsa_budget", "tsa_select", "tsa_gather_qkv", "tsa_attn",
              "tsa_scatter_residual", "tsa_layer"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = tsa.lib()
    for n in _declared():
        assert hasattr(lib, n), n
    assert set(_declared()) == set(tsa.EXPORTS)


def _d(B=1, L=4096, H=32, Hkv=8, d=128, dt=tsa.TSA_BF16):
    return tsa.Dims(B, L, H, Hkv, d, dt)


def test_workspace_size_host_query():
    n1 = tsa.workspace_size(_d(), 16)
    n2 = tsa.workspace_size(_d(L=8192), 16)
    assert 256 <= n1 < n2
    big = tsa.workspace_size(_d(), 16, layer=True)
    # the layer workspace holds Qh, Kh, Vh, Oh of [B, H, L, d] bf16
    assert big >= 4 * 32 * 4096 * 128 * 2 + n1
    assert tsa.workspace_size(_d(dt=tsa.TSA_F32, d=64), 16, layer=True) > 0


@pytest.mark.parametrize("kw,q", [(dict(d=96), 16), (dict(H=30, Hkv=8), 16), (dict(L=0), 16),
                                  (dict(B=0), 1), (dict(), 0), (dict(H=32, Hkv=1), 16),
                                  (dict(dt=7), 16), (dict(L=(1 << 21) + 1), 16)])
def test_workspace_size_rejects_bad_dims(kw, q):
    dm = _d(**kw)
    assert tsa.lib().tsa_workspace_size(ctypes.byref(dm), q) == 0


FAKE = 0x10000  # never dereferenced: every call below fails validation first
P = ctypes.c_void_p


def _score(dm, Q=FAKE, K=FAKE, q=16, scale=0.088, sh=FAKE, sl=FAKE, ws=FAKE * 16, wsb=1 << 30):
    return tsa.lib().tsa_score(ctypes.byref(dm), P(Q), P(K), q, scale, P(sh), P(sl), P(ws),
                               wsb, None)


def test_score_validation():
    dm = _d()
    assert _score(dm, Q=0) == 1                   # NULL
    assert _score(dm, K=FAKE + 8) == 2            # misaligned
    assert _score(dm, scale=0.0) == 1
    assert _score(dm, scale=float("nan")) == 1
    assert _score(dm, q=0) == 1
    assert _score(_d(H=64, Hkv=1), q=16) == 3     # G*q > 256
    assert _score(dm, wsb=100) == 4               # workspace too small
    assert _score(dm, ws=FAKE + 16) == 4          # workspace misaligned
    assert _score(_d(d=80)) == 3
    assert b"256" in tsa.lib().tsa_last_error() or True


def test_budget_and_select_validation():
    dm = _d()
    L = tsa.lib()
    assert L.tsa_budget(ctypes.byref(dm), P(FAKE), 1.0, P(FAKE), P(FAKE * 16), 4096, None) == 1
    assert L.tsa_budget(ctypes.byref(dm), P(FAKE), -0.1, P(FAKE), P(FAKE * 16), 4096, None) == 1
    assert L.tsa_budget(ctypes.byref(dm), P(FAKE), float("nan"), P(FAKE), P(FAKE * 16), 4096,
                        None) == 1
    assert L.tsa_budget(ctypes.byref(dm), P(0), 0.01, P(FAKE), P(FAKE * 16), 4096, None) == 1
    assert L.tsa_budget(ctypes.byref(dm), P(FAKE), 0.01, P(FAKE), P(FAKE * 16), 8, None) == 4
    assert L.tsa_select(ctypes.byref(dm), P(FAKE), P(FAKE + 4), P(FAKE), P(FAKE * 16), 4096,
                        None) == 2
    assert L.tsa_select(ctypes.byref(dm), P(FAKE), P(FAKE), P(0), P(FAKE * 16), 4096, None) == 1


def test_gather_attn_scatter_layer_validation():
    dm = _d()
    L = tsa.lib()
    f = [P(FAKE)] * 8
    assert L.tsa_gather_qkv(ctypes.byref(dm), P(0), *f[:7], P(FAKE * 16), 4096, None) == 1
    assert L.tsa_gather_qkv(ctypes.byref(dm), *f[:7], P(FAKE + 2), P(FAKE * 16), 4096, None) == 2
    assert L.tsa_gather_qkv(ctypes.byref(dm), *f[:8], P(FAKE * 16), 8, None) == 4
    assert L.tsa_attn(ctypes.byref(dm), P(FAKE), P(FAKE), P(FAKE), P(0), 0, 0.088, P(FAKE),
                      P(FAKE * 16), 4096, None) == 1      # compressed mode needs Lkeep
    assert L.tsa_attn(ctypes.byref(dm), P(FAKE), P(FAKE), P(FAKE), None, 1, -1.0, P(FAKE),
                      P(FAKE * 16), 4096, None) == 1
    assert L.tsa_scatter_residual(ctypes.byref(dm), P(FAKE), P(FAKE), P(0), P(FAKE), P(FAKE),
                                  None) == 1
    assert L.tsa_layer(ctypes.byref(dm), *[P(FAKE)] * 5, 1, 16, 1.5, 0.088, None, None, None,
                       None, P(FAKE * 16), 1 << 40, None, None) == 1
    assert L.tsa_layer(ctypes.byref(dm), *[P(FAKE)] * 5, 1, 16, 0.01, 0.088, None, None, None,
                       None, P(FAKE * 16), 1 << 20, None, None) == 4


def test_variant_validation():
    dm = _d()
    L = tsa.lib()
    n0 = tsa.kernel_launches()
    for s in (-0.1, 1.01, float("nan")):
        assert L.tsa_budget_fixed(ctypes.byref(dm), s, P(FAKE), None) == 1
    assert L.tsa_budget_fixed(ctypes.byref(dm), 0.3, P(0), None) == 1
    assert L.tsa_budget_fixed(ctypes.byref(_d(L=0)), 0.3, P(FAKE), None) == 1
    pool = lambda kind, width, out=FAKE * 64, wsb=1 << 30: L.tsa_pool_scores(
        ctypes.byref(dm), P(FAKE), kind, width, P(out), P(FAKE), P(FAKE * 16), wsb, None)
    assert pool(0, 3) == 1 and pool(3, 3) == 1 and pool(1, 4) == 1 and pool(2, -1) == 1
    assert pool(1, 257) == 3
    assert pool(1, 3, out=FAKE) == 1                    # output overlaps the input
    assert pool(1, 3, wsb=8) == 4
    opts = tsa.LayerOpts(7, 0.01, 0.0, 0, 1)              # unknown budget kind
    ex = lambda o: L.tsa_layer_ex(ctypes.byref(dm), *[P(FAKE)] * 5, 1, 16, ctypes.byref(o),
                                  0.088, None, None, None, None, P(FAKE * 16), 1 << 40, None,
                                  None)
    assert ex(opts) == 1
    assert ex(tsa.LayerOpts(1, 0.01, 1.5, 0, 1)) == 1    # sparsity out of range
    assert ex(tsa.LayerOpts(0, 0.01, 0.0, 2, 8)) == 1    # even pool width
    assert ex(tsa.LayerOpts(0, 0.01, 0.0, 1, 301)) == 3  # pool width above 255
    assert tsa.kernel_launches() == n0
    # workspace: the layer holds the pooled scores too
    assert tsa.workspace_size(dm, 16, layer=True) >= 2 * 4 * 32 * 4096 + 4 * 32 * 4096 * 128 * 2


def test_drift_validation():
    L = tsa.lib()
    n0 = tsa.kernel_launches()
    assert L.tsa_drift_workspace_size(0, 10) == 0 and L.tsa_drift_workspace_size(513, 10) == 0
    assert L.tsa_drift_workspace_size(32, 4096) >= 256 + 64 * 32 * 8
    dr = lambda N=4, T=100, D=256, dt=tsa.TSA_BF16, h=FAKE, eps=1e-6, delta=0.5, wsb=1 << 30: \
        L.tsa_drift(N, T, D, dt, P(h), eps, delta, P(FAKE), P(FAKE), P(FAKE * 16), wsb, None)
    assert dr(N=0) == 1 and dr(N=513) == 1 and dr(T=0) == 1
    assert dr(D=4) == 3 and dr(dt=7) == 3                 # 8 bytes per row, unknown dtype
    assert dr(eps=-1.0) == 1 and dr(delta=1.5) == 1 and dr(eps=float("nan")) == 1
    assert dr(h=0) == 1 and dr(h=FAKE + 4) == 2 and dr(wsb=16) == 4
    assert tsa.kernel_launches() == n0


def test_failed_validation_launches_nothing():
    n0 = tsa.kernel_launches()
    dm = _d()
    assert _score(dm, Q=0) == 1
    assert tsa.lib().tsa_select(ctypes.byref(dm), P(FAKE), P(FAKE), P(0), P(FAKE * 16), 4096,
                                None) == 1
    assert tsa.kernel_launches() == n0


def test_status_strings():
    L = tsa.lib()
    for code, name in tsa.STATUS.items():
        assert L.tsa_status_string(code).decode() == name
