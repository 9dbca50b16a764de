"""Python binding of libtsa: the same entry points as include/tsa.h.

Argument marshalling only: tensors become device pointers, torch's current
stream becomes the stream argument, and a non-OK status becomes a TSAError.
Every step of the layer runs in the CUDA library; if libtsa.so is missing the
first call raises instead of doing anything else.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libtsa.so")
_lib = None

TSA_F32, TSA_BF16 = 0, 1
STATUS = {0: "TSA_OK", 1: "TSA_ERR_INVALID_ARG", 2: "TSA_ERR_ALIGNMENT",
          3: "TSA_ERR_UNSUPPORTED", 4: "TSA_ERR_WORKSPACE", 5: "TSA_ERR_CUDA",
          6: "TSA_ERR_DEVICE_TIMEOUT", 7: "TSA_ERR_NONFINITE"}
EXPORTS = ("tsa_workspace_size", "tsa_layer_workspace_size", "tsa_score", "tsa_budget",
           "tsa_select", "tsa_gather_qkv", "tsa_attn", "tsa_scatter_residual", "tsa_layer",
           "tsa_get_device_status", "tsa_set_wait_limit", "tsa_status_string",
           "tsa_last_error", "tsa_score_fixed_scratch", "tsa_set_test_stall",
           "tsa_set_score_schedule", "tsa_kernel_launches", "tsa_budget_fixed", "tsa_pool_scores", "tsa_layer_ex",
           "tsa_drift_workspace_size", "tsa_drift", "tsa_attn_gather",
           "tsa_block_workspace_size", "tsa_block_select", "tsa_attn_block",
           "tsa_score_fixed_scratch_status", "tsa_score_fixed_scratch_forget",
           "tsa_score_partial", "tsa_layer_score_combine")
POOL_NONE, POOL_MAX, POOL_MEAN = 0, 1, 2
BUDGET_COVERAGE, BUDGET_FIXED = 0, 1


class TSAError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__("%s: %s" % (STATUS.get(status, status), msg))
        self.status = status


class Dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("L", ctypes.c_int32), ("H", ctypes.c_int32),
                ("Hkv", ctypes.c_int32), ("d", ctypes.c_int32), ("dtype", ctypes.c_int32)]


class LayerOpts(ctypes.Structure):
    """tsa_layer_opts of include/tsa.h."""
    _fields_ = [("budget", ctypes.c_int32), ("tau", ctypes.c_double),
                ("sparsity", ctypes.c_double), ("pool", ctypes.c_int32),
                ("pool_width", ctypes.c_int32), ("direct_gather", ctypes.c_int32),
                ("block_theta", ctypes.c_double)]


def lib():
    """Load libtsa.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError("libtsa.so is not built (python -m token_sparse_attention_dtc_b200.build)")
        L = ctypes.CDLL(_LIB_PATH)
        P, I32, SZ, D, F = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t, ctypes.c_double,
                            ctypes.c_float)
        DP = ctypes.POINTER(Dims)
        sig = {
            "tsa_workspace_size": (SZ, [DP, I32]),
            "tsa_layer_workspace_size": (SZ, [DP, I32]),
            "tsa_score": (I32, [DP, P, P, I32, F, P, P, P, SZ, P]),
            "tsa_budget": (I32, [DP, P, D, P, P, SZ, P]),
            "tsa_score_partial": (I32, [DP, P, P, I32, F, P, P, P, SZ, P]),
            "tsa_layer_score_combine": (I32, [DP, I32, P, P, P, SZ, P]),
            "tsa_select": (I32, [DP, P, P, P, P, SZ, P]),
            "tsa_gather_qkv": (I32, [DP, P, P, P, P, P, P, P, P, P, SZ, P]),
            "tsa_attn": (I32, [DP, P, P, P, P, I32, F, P, P, SZ, P]),
            "tsa_scatter_residual": (I32, [DP, P, P, P, P, P, P]),
            "tsa_layer": (I32, [DP, P, P, P, P, P, I32, I32, D, F, P, P, P, P, P, SZ, P, P]),
            "tsa_get_device_status": (I32, [P, P]),
            "tsa_set_wait_limit": (None, [ctypes.c_uint32]),
            "tsa_set_test_stall": (None, [I32]),
            "tsa_set_score_schedule": (None, [I32, I32]),
            "tsa_kernel_launches": (ctypes.c_uint64, []),
            "tsa_status_string": (ctypes.c_char_p, [I32]),
            "tsa_last_error": (ctypes.c_char_p, []),
            "tsa_score_fixed_scratch": (I32, [DP, P, P, I32, F, P, P, P]),
            "tsa_score_fixed_scratch_status": (I32, [P]),
            "tsa_score_fixed_scratch_forget": (None, []),
            "tsa_budget_fixed": (I32, [DP, D, P, P]),
            "tsa_attn_gather": (I32, [DP, P, P, P, P, P, F, P, P, P, SZ, P]),
            "tsa_block_workspace_size": (SZ, [DP]),
            "tsa_block_select": (I32, [DP, P, P, P, F, D, P, P, P, SZ, P]),
            "tsa_attn_block": (I32, [DP, P, P, P, P, P, F, P, P, SZ, P]),
            "tsa_drift_workspace_size": (SZ, [I32, ctypes.c_int64]),
            "tsa_drift": (I32, [I32, ctypes.c_int64, I32, I32, P, D, D, P, P, P, SZ, P]),
            "tsa_pool_scores": (I32, [DP, P, I32, I32, P, P, P, SZ, P]),
            "tsa_layer_ex": (I32, [DP, P, P, P, P, P, I32, I32, ctypes.POINTER(LayerOpts), F,
                                   P, P, P, P, P, SZ, P, P]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype, f.argtypes = res, args
        _lib = L
    return _lib


def _check(status: int):
    if status != 0:
        raise TSAError(status, lib().tsa_last_error().decode())


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


def dims(Q: torch.Tensor, K: torch.Tensor) -> Dims:
    """Dims of Q [B, L, H, d] and K [B, L, Hkv, d]."""
    B, L, H, d = Q.shape
    if Q.dtype == torch.bfloat16:
        dt = TSA_BF16
    elif Q.dtype == torch.float32:
        dt = TSA_F32
    else:
        raise ValueError("Q must be bf16 or fp32")
    return Dims(B, L, H, K.shape[2], d, dt)


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)


def workspace_size(dm: Dims, q: int, layer: bool = False) -> int:
    f = lib().tsa_layer_workspace_size if layer else lib().tsa_workspace_size
    n = f(ctypes.byref(dm), q)
    if n == 0:
        raise TSAError(1, lib().tsa_last_error().decode())
    return n


def workspace(dm: Dims, q: int, layer: bool = False, device=None) -> torch.Tensor:
    """A zero-filled workspace (torch allocations are 256-byte aligned)."""
    return torch.zeros(workspace_size(dm, q, layer), dtype=torch.uint8, device=device or "cuda")


def tsa_score(Q, K, q: int, scale: float | None = None, s_h=None, s_l=None, ws=None,
              stream=None):
    dm = dims(Q, K)
    _need_cuda(Q, K)
    if s_h is None:
        s_h = torch.empty(dm.B, dm.H, dm.L, dtype=torch.float32, device=Q.device)
    if s_l is None:
        s_l = torch.empty(dm.B, dm.L, dtype=torch.float32, device=Q.device)
    if ws is None:
        ws = workspace(dm, q, device=Q.device)
    _check(lib().tsa_score(ctypes.byref(dm), _p(Q), _p(K), q,
                           default_scale(dm.d) if scale is None else scale, _p(s_h), _p(s_l),
                           _p(ws), ws.numel(), _stream(stream)))
    return s_h, s_l


def tsa_score_fixed_scratch(Q, K, q: int, scale: float | None = None, s_h=None, s_l=None,
                            stream=None):
    """tsa_score without a workspace argument: the library's fixed device scratch is used
    (for callers that cannot allocate device memory at call time)."""
    dm = dims(Q, K)
    _need_cuda(Q, K)
    if s_h is None:
        s_h = torch.empty(dm.B, dm.H, dm.L, dtype=torch.float32, device=Q.device)
    if s_l is None:
        s_l = torch.empty(dm.B, dm.L, dtype=torch.float32, device=Q.device)
    _check(lib().tsa_score_fixed_scratch(ctypes.byref(dm), _p(Q), _p(K), q,
                                         default_scale(dm.d) if scale is None else scale,
                                         _p(s_h), _p(s_l), _stream(stream)))
    return s_h, s_l


def tsa_score_fixed_scratch_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the error word of the fixed scratch
    on the current device."""
    return int(lib().tsa_score_fixed_scratch_status(_stream(stream)))


def tsa_score_partial(Q, K, q: int, scale: float | None = None, s_h=None, u_part=None,
                      ws=None, stream=None):
    """Scores of this shard's heads: returns (s_h [B, H, L], u_part [B, L]), u_part the
    unnormalised sum of s_h over the shard's heads."""
    dm = dims(Q, K)
    _need_cuda(Q, K)
    if s_h is None:
        s_h = torch.empty(dm.B, dm.H, dm.L, dtype=torch.float32, device=Q.device)
    if u_part is None:
        u_part = torch.empty(dm.B, dm.L, dtype=torch.float32, device=Q.device)
    if ws is None:
        ws = workspace(dm, q, device=Q.device)
    _check(lib().tsa_score_partial(ctypes.byref(dm), _p(Q), _p(K), q,
                                   default_scale(dm.d) if scale is None else scale, _p(s_h),
                                   _p(u_part), _p(ws), ws.numel(), _stream(stream)))
    return s_h, u_part


def tsa_layer_score_combine(dm: Dims, u_parts, s_l=None, ws=None, stream=None):
    """s_l [B, L] from the partials u_parts [nparts, B, L] (summed in index order)."""
    _need_cuda(u_parts)
    if s_l is None:
        s_l = torch.empty(dm.B, dm.L, dtype=torch.float32, device=u_parts.device)
    if ws is None:
        ws = workspace(dm, 1, device=u_parts.device)
    _check(lib().tsa_layer_score_combine(ctypes.byref(dm), int(u_parts.shape[0]), _p(u_parts),
                                         _p(s_l), _p(ws), ws.numel(), _stream(stream)))
    return s_l


def tsa_budget(dm: Dims, s_l, tau: float, Lkeep=None, ws=None, stream=None):
    _need_cuda(s_l)
    if Lkeep is None:
        Lkeep = torch.empty(dm.B, dtype=torch.int32, device=s_l.device)
    if ws is None:
        ws = workspace(dm, 1, device=s_l.device)
    _check(lib().tsa_budget(ctypes.byref(dm), _p(s_l), float(tau), _p(Lkeep), _p(ws),
                            ws.numel(), _stream(stream)))
    return Lkeep


def tsa_select(dm: Dims, s_h, Lkeep, idx=None, ws=None, stream=None):
    _need_cuda(s_h, Lkeep)
    if idx is None:
        idx = torch.empty(dm.B, dm.H, dm.L, dtype=torch.int32, device=s_h.device)
    if ws is None:
        ws = workspace(dm, 1, device=s_h.device)
    _check(lib().tsa_select(ctypes.byref(dm), _p(s_h), _p(Lkeep), _p(idx), _p(ws), ws.numel(),
                            _stream(stream)))
    return idx


def tsa_gather_qkv(Q, K, V, idx, Lkeep, Qh=None, Kh=None, Vh=None, ws=None, stream=None):
    dm = dims(Q, K)
    _need_cuda(Q, K, V, idx, Lkeep)
    shape = (dm.B, dm.H, dm.L, dm.d)
    Qh = torch.empty(shape, dtype=Q.dtype, device=Q.device) if Qh is None else Qh
    Kh = torch.empty(shape, dtype=Q.dtype, device=Q.device) if Kh is None else Kh
    Vh = torch.empty(shape, dtype=Q.dtype, device=Q.device) if Vh is None else Vh
    if ws is None:
        ws = workspace(dm, 1, device=Q.device)
    _check(lib().tsa_gather_qkv(ctypes.byref(dm), _p(Q), _p(K), _p(V), _p(idx), _p(Lkeep),
                                _p(Qh), _p(Kh), _p(Vh), _p(ws), ws.numel(), _stream(stream)))
    return Qh, Kh, Vh


def tsa_attn(dm: Dims, Qh, Kh, Vh, Lkeep=None, dense: bool = False, scale: float | None = None,
             Oh=None, ws=None, stream=None):
    _need_cuda(Qh, Kh, Vh, Lkeep)
    if Oh is None:
        Oh = torch.empty_like(Qh)
    if ws is None:
        ws = workspace(dm, 1, device=Qh.device)
    _check(lib().tsa_attn(ctypes.byref(dm), _p(Qh), _p(Kh), _p(Vh), _p(Lkeep), int(dense),
                          default_scale(dm.d) if scale is None else scale, _p(Oh), _p(ws),
                          ws.numel(), _stream(stream)))
    return Oh


def tsa_scatter_residual(dm: Dims, Oh, idx, Lkeep, X, Y=None, stream=None):
    _need_cuda(Oh, idx, Lkeep, X)
    if Y is None:
        Y = torch.empty_like(X)
    _check(lib().tsa_scatter_residual(ctypes.byref(dm), _p(Oh), _p(idx), _p(Lkeep), _p(X),
                                      _p(Y), _stream(stream)))
    return Y


def tsa_drift(h, eps: float = 1e-6, delta: float = 0.5, ws=None, stream=None):
    """Drift R [N] (fp64) and sparse-layer mask [N] (int32) of hidden states h
    [N + 1, T, D] (bf16 or fp32, on the GPU)."""
    _need_cuda(h)
    if h.dim() != 3 or not h.is_contiguous():
        raise ValueError("h must be a contiguous [N + 1, T, D] tensor")
    N, T, D = h.shape[0] - 1, h.shape[1], h.shape[2]
    dt = TSA_BF16 if h.dtype == torch.bfloat16 else TSA_F32
    R = torch.empty(max(N, 0), dtype=torch.float64, device=h.device)
    mask = torch.empty(max(N, 0), dtype=torch.int32, device=h.device)
    if ws is None:
        n = lib().tsa_drift_workspace_size(N, T)
        ws = torch.zeros(max(n, 256), dtype=torch.uint8, device=h.device)
    _check(lib().tsa_drift(N, T, D, dt, _p(h), float(eps), float(delta), _p(R), _p(mask),
                           _p(ws), ws.numel(), _stream(stream)))
    return R, mask


def tsa_attn_gather(Q, K, V, idx, Lkeep, X, Y=None, scale: float | None = None, ws=None,
                    stream=None):
    """Fused compress + attention + decompress: returns Y (= X + Decompress(Ô))."""
    dm = dims(Q, K)
    _need_cuda(Q, K, V, idx, Lkeep, X)
    if Y is None:
        Y = torch.empty_like(X)
    if ws is None:
        ws = workspace(dm, 1, device=Q.device)
    _check(lib().tsa_attn_gather(ctypes.byref(dm), _p(Q), _p(K), _p(V), _p(idx), _p(Lkeep),
                                 default_scale(dm.d) if scale is None else scale, _p(X), _p(Y),
                                 _p(ws), ws.numel(), _stream(stream)))
    return Y


def block_shape(dm: Dims):
    """(NP, NB, NW) of the block-sparse pattern for these dims."""
    NP, NB = (dm.L + 255) // 256, (dm.L + 127) // 128
    return NP, NB, (NB + 31) // 32


def tsa_block_select(dm: Dims, Qh, Kh, Lkeep, theta: float, scale: float | None = None,
                     logits: bool = True, ws=None, stream=None):
    """Block logits [B, H, NP, NB] (or None) and kept-block mask [B, H, NP, NW] uint32."""
    _need_cuda(Qh, Kh, Lkeep)
    NP, NB, NW = block_shape(dm)
    z = torch.empty(dm.B, dm.H, NP, NB, dtype=torch.float32, device=Qh.device) if logits else None
    mask = torch.empty(dm.B, dm.H, NP, NW, dtype=torch.int32, device=Qh.device)
    if ws is None:
        ws = torch.zeros(max(256, lib().tsa_block_workspace_size(ctypes.byref(dm))),
                         dtype=torch.uint8, device=Qh.device)
    _check(lib().tsa_block_select(ctypes.byref(dm), _p(Qh), _p(Kh), _p(Lkeep),
                                  default_scale(dm.d) if scale is None else scale, float(theta),
                                  _p(z), _p(mask), _p(ws), ws.numel(), _stream(stream)))
    return z, mask


def tsa_attn_block(dm: Dims, Qh, Kh, Vh, Lkeep, mask, scale: float | None = None, Oh=None,
                   ws=None, stream=None):
    """Compressed attention restricted to the kept blocks of mask."""
    _need_cuda(Qh, Kh, Vh, Lkeep, mask)
    if Oh is None:
        Oh = torch.empty_like(Qh)
    if ws is None:
        ws = workspace(dm, 1, device=Qh.device)
    _check(lib().tsa_attn_block(ctypes.byref(dm), _p(Qh), _p(Kh), _p(Vh), _p(Lkeep), _p(mask),
                                default_scale(dm.d) if scale is None else scale, _p(Oh), _p(ws),
                                ws.numel(), _stream(stream)))
    return Oh


def tsa_budget_fixed(dm: Dims, sparsity: float, Lkeep=None, device=None, stream=None):
    """Fixed-ratio budget: Lkeep[b] = L - floor(sparsity * L)."""
    if Lkeep is None:
        Lkeep = torch.empty(dm.B, dtype=torch.int32, device=device or "cuda")
    _need_cuda(Lkeep)
    _check(lib().tsa_budget_fixed(ctypes.byref(dm), float(sparsity), _p(Lkeep), _stream(stream)))
    return Lkeep


def tsa_pool_scores(dm: Dims, s_h, kind: int, width: int, s_h_out=None, s_l_out=None, ws=None,
                    stream=None):
    """Token-axis max / mean pooling of s_h [B, H, L]; returns (pooled s_h, s_l)."""
    _need_cuda(s_h)
    if s_h_out is None:
        s_h_out = torch.empty_like(s_h)
    if s_l_out is None:
        s_l_out = torch.empty(dm.B, dm.L, dtype=torch.float32, device=s_h.device)
    if ws is None:
        ws = workspace(dm, 1, device=s_h.device)
    _check(lib().tsa_pool_scores(ctypes.byref(dm), _p(s_h), int(kind), int(width), _p(s_h_out),
                                 _p(s_l_out), _p(ws), ws.numel(), _stream(stream)))
    return s_h_out, s_l_out


def tsa_layer(Q, K, V, X, Y=None, is_sparse: bool = True, q: int = 16, tau: float = 0.005,
              scale: float | None = None, s_h=None, s_l=None, Lkeep=None, idx=None, ws=None,
              stream=None, stage_events=None, sparsity: float | None = None,
              pool: int = POOL_NONE, pool_width: int = 1, direct: bool = False,
              block_theta: float | None = None):
    """One Token Sparse Attention layer: returns Y = X + Decompress(Ô) (or the dense layer).
    sparsity (fixed-ratio budget instead of tau) and pool / pool_width (pooled head
    scores) and direct (fused compress + attention + decompress) select the variants of
    tsa_layer_ex."""
    dm = dims(Q, K)
    _need_cuda(Q, K, V, X, Y, s_h, s_l, Lkeep, idx)
    if Y is None:
        Y = torch.empty_like(X)
    if ws is None:
        ws = workspace(dm, q, layer=True, device=Q.device)
    ev = None
    if stage_events is not None:
        ev = (ctypes.c_void_p * 7)(*[ctypes.c_void_p(e.cuda_event) for e in stage_events])
    sc = default_scale(dm.d) if scale is None else scale
    if sparsity is None and pool == POOL_NONE and not direct and block_theta is None:
        _check(lib().tsa_layer(ctypes.byref(dm), _p(Q), _p(K), _p(V), _p(X), _p(Y),
                               int(is_sparse), q, float(tau), sc, _p(s_h), _p(s_l), _p(Lkeep),
                               _p(idx), _p(ws), ws.numel(), _stream(stream), ev))
        return Y
    o = LayerOpts(BUDGET_COVERAGE if sparsity is None else BUDGET_FIXED, float(tau),
                  0.0 if sparsity is None else float(sparsity), int(pool), int(pool_width),
                  int(bool(direct)), -1.0 if block_theta is None else float(block_theta))
    _check(lib().tsa_layer_ex(ctypes.byref(dm), _p(Q), _p(K), _p(V), _p(X), _p(Y),
                              int(is_sparse), q, ctypes.byref(o), sc, _p(s_h), _p(s_l),
                              _p(Lkeep), _p(idx), _p(ws), ws.numel(), _stream(stream), ev))
    return Y


def tsa_get_device_status(ws, stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error word."""
    st = lib().tsa_get_device_status(_p(ws), _stream(stream))
    return int(st)


def tsa_set_wait_limit(microseconds: int):
    lib().tsa_set_wait_limit(int(microseconds))


def kernel_launches() -> int:
    """Kernels the library has launched so far in this process (host-side counter)."""
    return int(lib().tsa_kernel_launches())


def tsa_set_test_stall(on: bool):
    """Failure-path test hook (see include/tsa.h)."""
    lib().tsa_set_test_stall(1 if on else 0)


def tsa_set_score_schedule(wave, max_groups_per_wave: int = 0):
    """bf16 scoring schedule: 0 / False the automatic choice (the default), 1 / True the
    wave-scheduled kernel wherever it applies, 2 / "single" the single-wave kernel
    everywhere; max_groups_per_wave > 0 caps the KV groups of one wave.  See
    include/tsa.h."""
    mode = 2 if wave == "single" else (1 if wave is True else int(wave))
    lib().tsa_set_score_schedule(mode, int(max_groups_per_wave))
