"""CPU oracle for the Token Sparse Attention layer.

TEST INFRASTRUCTURE ONLY.  The plain fp64 C code in ``tsa_oracle.c`` restates
the method of "Token Sparse Attention: Efficient Long-Context Inference with
Interleaved Token Selection" step by step (papernotes.org notes, 方法详解 and
关键设计 1-2; bxzpzcl.cn post §1.1 and §2.1; gist.science summary §2).  Only the
test suite, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this module.  It shares nothing with the CUDA library.

Inputs are numpy arrays (or CPU torch tensors) in one of two storage types:
fp32, or bf16 given as raw uint16 bits.  Every result is float64 except the
integer budget and index outputs.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tsa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile tsa_oracle.c into liboracle.so beside it (gcc, -O2, pthreads)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-pthread", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P, I, D, L = ctypes.c_void_p, ctypes.c_int, ctypes.c_double, ctypes.c_long
        lib.orc_score.argtypes = [I, I, I, I, I, I, I, P, P, D, P, P, I]
        lib.orc_budget.argtypes = [I, I, P, D, P, P]
        lib.orc_select.argtypes = [I, I, I, P, P, P]
        lib.orc_attend_rows.argtypes = [I, I, I, I, I, I, P, P, P, P, P, D, L, P, P, I]
        lib.orc_decompress_residual.argtypes = [I, I, I, I, I, P, P, P, P, P, P]
        lib.orc_budget_fixed.argtypes = [I, I, D, P]
        lib.orc_pool.argtypes = [I, I, I, P, I, I, P, P]
        lib.orc_drift.argtypes = [I, L, I, I, P, D, P]
        lib.orc_drift_mask.argtypes = [I, P, D, P]
        lib.orc_block_logits.argtypes = [I, I, I, I, I, I, P, P, P, P, D, P]
        lib.orc_block_select.argtypes = [I, I, I, P, P, ctypes.c_float, P]
        lib.orc_attend_block_rows.argtypes = [I, I, I, I, I, I, P, P, P, P, P, P, D, P, L, P]
        for f in ("orc_score", "orc_budget", "orc_select", "orc_attend_rows",
                  "orc_decompress_residual", "orc_budget_fixed", "orc_pool", "orc_drift",
                  "orc_drift_mask", "orc_block_logits", "orc_block_select",
                  "orc_attend_block_rows"):
            getattr(lib, f).restype = ctypes.c_int
        _lib = lib
    return _lib


def _np(x):
    """numpy view of a CPU array/tensor; bf16 tensors become their uint16 bits."""
    try:
        import torch

        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                return x.view(torch.int16).numpy().view(np.uint16)
            return x.numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(x)


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return 0
    if a.dtype == np.uint16:
        return 1
    raise TypeError("oracle inputs must be float32 or bf16 (uint16 bits), got %s" % a.dtype)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _threads(nthreads):
    return int(nthreads or os.cpu_count() or 1)


def score(Q, K, q: int, scale: float | None = None, nthreads: int | None = None):
    """Dynamic Token Coverage scores.

    Q: [B, L, H, d] (only the last min(q, L) rows are read), K: [B, L, Hkv, d].
    Returns (s_h [B, H, L] float64, s_l [B, L] float64).
    """
    Qn, Kn = _np(Q), _np(K)
    B, L, H, d = Qn.shape
    Hkv = Kn.shape[2]
    qe = min(q, L)
    Qr = np.ascontiguousarray(Qn[:, L - qe:])
    code = _dtype_code(Qn)
    assert _dtype_code(Kn) == code
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    s_h = np.zeros((B, H, L), np.float64)
    s_l = np.zeros((B, L), np.float64)
    rc = _load().orc_score(B, L, H, Hkv, d, code, q, _ptr(Qr), _ptr(Kn), float(scale),
                           _ptr(s_h), _ptr(s_l), _threads(nthreads))
    if rc:
        raise ValueError("orc_score rejected its arguments (%d)" % rc)
    return s_h, s_l


def budget(s_l, tau: float):
    """Coverage budget on fp32 s_l [B, L]; returns (Lkeep int32 [B], real_disagree)."""
    s = np.ascontiguousarray(_np(s_l), dtype=np.float32)
    B, L = s.shape
    out = np.zeros(B, np.int32)
    dis = np.zeros(1, np.int32)
    rc = _load().orc_budget(B, L, _ptr(s), float(tau), _ptr(out), _ptr(dis))
    if rc:
        raise ValueError("orc_budget rejected its arguments (%d)" % rc)
    return out, int(dis[0])


def budget_fixed(B: int, L: int, sparsity: float):
    """Fixed-ratio budget (ablation): L' = L - floor(sparsity * L) for every batch element."""
    out = np.zeros(B, np.int32)
    rc = _load().orc_budget_fixed(int(B), int(L), float(sparsity), _ptr(out))
    if rc:
        raise ValueError("orc_budget_fixed rejected its arguments (%d)" % rc)
    return out


POOL_MAX, POOL_MEAN = 1, 2


def pool(s_h, kind: int, width: int):
    """Token-axis pooling of head scores s_h [B, H, L] (any float dtype, taken exactly);
    kind POOL_MAX or POOL_MEAN over the clipped window of odd `width`.  Returns
    (pooled fp64 [B, H, L], s_l fp64 [B, L])."""
    s = np.ascontiguousarray(_np(s_h), dtype=np.float64)
    B, H, L = s.shape
    out = np.zeros((B, H, L), np.float64)
    sl = np.zeros((B, L), np.float64)
    rc = _load().orc_pool(B, H, L, _ptr(s), int(kind), int(width), _ptr(out), _ptr(sl))
    if rc:
        raise ValueError("orc_pool rejected its arguments (%d)" % rc)
    return out, sl


def drift(h, eps: float = 1e-6):
    """Per-layer drift R [N] (fp64) of hidden states h [N + 1, T, D] (fp32 or bf16)."""
    a = _np(h)
    N1, T, D = a.shape
    a = np.ascontiguousarray(a)
    R = np.zeros(N1 - 1, np.float64)
    rc = _load().orc_drift(N1 - 1, T, D, _dtype_code(a), _ptr(a), float(eps), _ptr(R))
    if rc:
        raise ValueError("orc_drift rejected its arguments (%d)" % rc)
    return R


def drift_mask(R, delta: float = 0.5):
    """Sparse-layer mask int32 [N]: 1 where rank(R_l) / N <= delta."""
    r = np.ascontiguousarray(_np(R), dtype=np.float64)
    mask = np.zeros(len(r), np.int32)
    rc = _load().orc_drift_mask(len(r), _ptr(r), float(delta), _ptr(mask))
    if rc:
        raise ValueError("orc_drift_mask rejected its arguments (%d)" % rc)
    return mask


def block_logits(Q, K, idx, Lkeep, scale: float | None = None):
    """Block logits z [B, H, ceil(L/256), ceil(L/128)] fp64 of the block-sparse pattern
    (NaN where a pair or block does not exist)."""
    q, k = _np(Q), _np(K)
    B, L, H, d = q.shape
    Hkv = k.shape[2]
    ix = np.ascontiguousarray(_np(idx), dtype=np.int32)
    lk = np.ascontiguousarray(_np(Lkeep), dtype=np.int32)
    z = np.zeros((B, H, (L + 255) // 256, (L + 127) // 128), np.float64)
    sc = 1.0 / np.sqrt(d) if scale is None else scale
    rc = _load().orc_block_logits(B, L, H, Hkv, d, _dtype_code(q), _ptr(q), _ptr(k), _ptr(ix),
                                  _ptr(lk), float(sc), _ptr(z))
    if rc:
        raise ValueError("orc_block_logits rejected its arguments (%d)" % rc)
    return z


def block_select(z, Lkeep, theta: float):
    """Kept blocks uint8 [B, H, NP, NB] from fp32 block logits z (fp32 threshold)."""
    zz = np.ascontiguousarray(_np(z), dtype=np.float32)
    B, H, NP, NB = zz.shape
    lk = np.ascontiguousarray(_np(Lkeep), dtype=np.int32)
    keep = np.zeros((B, H, NP, NB), np.uint8)
    L = NB * 128
    rc = _load().orc_block_select(B, H, L, _ptr(lk), _ptr(zz), ctypes.c_float(theta), _ptr(keep))
    if rc:
        raise ValueError("orc_block_select rejected its arguments (%d)" % rc)
    return keep


def attend_block_rows(Q, K, V, idx, Lkeep, keep, rows, scale: float | None = None):
    """Block-sparse attention rows Ô[b, h, i] for rows [(b, h, i), ...]; fp64 [n, d]."""
    q, k, v = _np(Q), _np(K), _np(V)
    B, L, H, d = q.shape
    ix = np.ascontiguousarray(_np(idx), dtype=np.int32)
    lk = np.ascontiguousarray(_np(Lkeep), dtype=np.int32)
    kp = np.ascontiguousarray(keep, dtype=np.uint8)
    assert kp.shape[2:] == ((L + 255) // 256, (L + 127) // 128)
    r = np.ascontiguousarray(np.asarray(rows, np.int32).reshape(-1, 3))
    out = np.zeros((len(r), d), np.float64)
    sc = 1.0 / np.sqrt(d) if scale is None else scale
    rc = _load().orc_attend_block_rows(B, L, H, k.shape[2], d, _dtype_code(q), _ptr(q), _ptr(k),
                                       _ptr(v), _ptr(ix), _ptr(lk), _ptr(kp), float(sc), _ptr(r),
                                       len(r), _ptr(out))
    if rc:
        raise ValueError("orc_attend_block_rows rejected its arguments (%d)" % rc)
    return out


def select(s_h, Lkeep):
    """Per-head top-L' on fp32 s_h [B, H, L]; returns idx int32 [B, H, L]
    (kept tokens ascending, then the rest ascending)."""
    s = np.ascontiguousarray(_np(s_h), dtype=np.float32)
    B, H, L = s.shape
    lk = np.ascontiguousarray(_np(Lkeep), dtype=np.int32)
    idx = np.zeros((B, H, L), np.int32)
    rc = _load().orc_select(B, H, L, _ptr(s), _ptr(lk), _ptr(idx))
    if rc:
        raise ValueError("orc_select rejected its arguments (%d)" % rc)
    return idx


def attend_rows(Q, K, V, idx, Lkeep, rows, scale: float | None = None,
                nthreads: int | None = None):
    """Compressed causal attention for the requested (b, h, i) rows.

    idx None means identity (dense attention); Lkeep None means L' = L.
    Returns float64 [n_rows, d].
    """
    Qn, Kn, Vn = _np(Q), _np(K), _np(V)
    B, L, H, d = Qn.shape
    Hkv = Kn.shape[2]
    code = _dtype_code(Qn)
    assert _dtype_code(Kn) == code and _dtype_code(Vn) == code
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int32).reshape(-1, 3))
    out = np.zeros((r.shape[0], d), np.float64)
    idx_keep = None if idx is None else np.ascontiguousarray(_np(idx), dtype=np.int32)
    ip = _ptr(idx_keep) if idx_keep is not None else None
    lk = None if Lkeep is None else np.ascontiguousarray(_np(Lkeep), dtype=np.int32)
    rc = _load().orc_attend_rows(B, L, H, Hkv, d, code, _ptr(Qn), _ptr(Kn), _ptr(Vn),
                                 ip, _ptr(lk) if lk is not None else None, float(scale),
                                 r.shape[0], _ptr(r), _ptr(out), _threads(nthreads))
    if rc:
        raise ValueError("orc_attend_rows rejected its arguments (%d)" % rc)
    return out


def attend(Q, K, V, idx, Lkeep, scale: float | None = None, nthreads: int | None = None):
    """All rows: returns Oh float64 [B, H, L, d]; rows i >= Lkeep[b] are zero."""
    Qn = _np(Q)
    B, L, H, d = Qn.shape
    lk = np.full(B, L, np.int32) if Lkeep is None else np.asarray(_np(Lkeep), np.int32)
    rows = [(b, h, i) for b in range(B) for h in range(H) for i in range(int(lk[b]))]
    out = np.zeros((B, H, L, d), np.float64)
    if rows:
        vals = attend_rows(Q, K, V, idx, Lkeep, rows, scale, nthreads)
        r = np.asarray(rows)
        out[r[:, 0], r[:, 1], r[:, 2]] = vals
    return out


def decompress_residual(Oh, idx, Lkeep, X):
    """Y = X + Decompress(Ô).  Oh float64 [B, H, L, d]; X [B, L, H*d].

    Returns (O_dec float64 [B, L, H*d], Y float64 [B, L, H*d]).
    """
    Xn = _np(X)
    B, L, HD = Xn.shape
    Ohn = np.ascontiguousarray(Oh, dtype=np.float64)
    H, d = Ohn.shape[1], Ohn.shape[3]
    assert H * d == HD
    ip = None
    if idx is not None:
        idx_keep = np.ascontiguousarray(_np(idx), dtype=np.int32)
        ip = _ptr(idx_keep)
    lk = None if Lkeep is None else np.ascontiguousarray(_np(Lkeep), dtype=np.int32)
    O = np.zeros((B, L, HD), np.float64)
    Y = np.zeros((B, L, HD), np.float64)
    rc = _load().orc_decompress_residual(B, L, H, d, _dtype_code(Xn), _ptr(Ohn), ip,
                                         _ptr(lk) if lk is not None else None, _ptr(Xn),
                                         _ptr(O), _ptr(Y))
    if rc:
        raise ValueError("orc_decompress_residual rejected its arguments (%d)" % rc)
    return O, Y


def layer(Q, K, V, X, q: int, tau: float, is_sparse: bool = True,
          nthreads: int | None = None):
    """The whole layer on the oracle's own arithmetic (small sizes only).

    Scores are rounded to fp32 before the budget and selection, as the
    integer decisions are defined on fp32 scores.
    Returns a dict with s_h, s_l, Lkeep, idx, Oh, O_dec, Y.
    """
    Qn = _np(Q)
    B, L, H, d = Qn.shape
    if not is_sparse:
        Oh = attend(Q, K, V, None, None, nthreads=nthreads)
        O_dec, Y = decompress_residual(Oh, None, None, X)
        return dict(Oh=Oh, O_dec=O_dec, Y=Y)
    s_h, s_l = score(Q, K, q, nthreads=nthreads)
    Lkeep, _ = budget(s_l.astype(np.float32), tau)
    idx = select(s_h.astype(np.float32), Lkeep)
    Oh = attend(Q, K, V, idx, Lkeep, nthreads=nthreads)
    O_dec, Y = decompress_residual(Oh, idx, Lkeep, X)
    return dict(s_h=s_h, s_l=s_l, Lkeep=Lkeep, idx=idx, Oh=Oh, O_dec=O_dec, Y=Y)
