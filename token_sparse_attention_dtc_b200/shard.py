"""One Token Sparse Attention layer sharded by KV group across GPUs (one process per GPU,
torch.distributed over NCCL for the one exchange).

The layer score couples the heads only through u[t] = sum_h s_h[h, t] (bxzpzcl.cn post
§2.1 层级预算分配; papernotes.org notes 关键设计 2).  Rank r holds a contiguous range of
KV groups: their query heads' Q [B, L, H_r, d], their K and V [B, L, Hkv_r, d] and
their columns of X and Y [B, L, H_r * d].  It scores its heads, all-gathers the partial
u of every rank, combines them in rank order on the device (the same s_l, bit for bit,
on every rank), and runs the budget, selection, compress, attention and decompress on
its own heads.  Every step of the method runs in libtsa; this module only moves the
partials between ranks.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import tsa


def kv_group_range(Hkv: int, rank: int, world: int) -> tuple[int, int]:
    """KV groups [kv0, kv1) of `rank`: contiguous, sizes differing by at most one."""
    if not 0 <= rank < world or world < 1:
        raise ValueError("rank %d outside a world of %d" % (rank, world))
    if world > Hkv:
        raise ValueError("%d ranks for %d KV groups: some rank would hold none" % (world, Hkv))
    per, rem = divmod(Hkv, world)
    kv0 = rank * per + min(rank, rem)
    return kv0, kv0 + per + (1 if rank < rem else 0)


def head_range(H: int, Hkv: int, rank: int, world: int) -> tuple[int, int]:
    """Query heads [h0, h1) of `rank` (those of its KV groups)."""
    G = H // Hkv
    kv0, kv1 = kv_group_range(Hkv, rank, world)
    return kv0 * G, kv1 * G


def exchange_partials(u_part: torch.Tensor, group=None) -> torch.Tensor:
    """All-gather every rank's partial layer score: returns [world, *u_part.shape], rank
    r's partial at index r, identical on every rank."""
    world = dist.get_world_size(group)
    u_part = u_part.contiguous()
    if dist.get_backend(group) == "nccl":
        out = torch.empty((world,) + tuple(u_part.shape), dtype=u_part.dtype,
                          device=u_part.device)
        dist.all_gather_into_tensor(out, u_part, group=group)
        return out
    parts = [torch.empty_like(u_part) for _ in range(world)]
    dist.all_gather(parts, u_part, group=group)
    return torch.stack(parts)


def sharded_layer(Q, K, V, X, Y=None, q: int = 16, tau: float = 0.005,
                  scale: float | None = None, group=None, ws=None, stream=None):
    """This rank's part of one sparse layer.  Q, K, V, X hold this rank's heads (see the
    module docstring); returns (Y, dict(s_h, s_l, Lkeep, idx)) with Y = this rank's
    columns of X + Decompress(Ô).  The budget Lkeep is the same on every rank."""
    dm = tsa.dims(Q, K)
    if ws is None:
        ws = tsa.workspace(dm, q, device=Q.device)
    s_h, u_part = tsa.tsa_score_partial(Q, K, q, scale=scale, ws=ws, stream=stream)
    parts = exchange_partials(u_part, group)
    s_l = tsa.tsa_layer_score_combine(dm, parts, ws=ws, stream=stream)
    Lk = tsa.tsa_budget(dm, s_l, tau, ws=ws, stream=stream)
    idx = tsa.tsa_select(dm, s_h, Lk, ws=ws, stream=stream)
    Qh, Kh, Vh = tsa.tsa_gather_qkv(Q, K, V, idx, Lk, ws=ws, stream=stream)
    Oh = tsa.tsa_attn(dm, Qh, Kh, Vh, Lk, scale=scale, ws=ws, stream=stream)
    Y = tsa.tsa_scatter_residual(dm, Oh, idx, Lk, X, Y, stream=stream)
    return Y, dict(s_h=s_h, s_l=s_l, Lkeep=Lk, idx=idx)
