"""Head sharding across the GPUs of one node.

Every (sequence, head) slice of exact attention is independent of every other, so
the heads of a batch can be partitioned across the GPUs of a node (codechina FlashAttention
article, §6.3 multi-GPU scaling: partition by attention heads, NCCL for the
communication between GPUs).  Each rank runs this package's kernels on its own
contiguous range of heads; the attention itself needs no collective.  Only a caller
that wants every head's output on every rank gathers the shards (``gather_heads``,
one ``all_gather`` over the process group: NCCL over NVLink on GPUs, gloo on CPU).

Nothing here computes attention: the local calls go to the CUDA kernels through
the C ABI, like every other entry point of the package.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch


def head_range(H: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous heads [h0, h1) of ``rank``: H split as evenly as possible, the
    first H % world ranks taking one head more."""
    if H < 1 or world < 1 or not (0 <= rank < world):
        raise ValueError(f"bad partition request H={H} world={world} rank={rank}")
    base, extra = divmod(H, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def local_heads(x: torch.Tensor, world: int, rank: int) -> torch.Tensor:
    """This rank's heads of a dense [B, H, ...] tensor, contiguous (the kernels take
    contiguous [B, H_local, N, d] buffers)."""
    h0, h1 = head_range(x.shape[1], world, rank)
    return x[:, h0:h1].contiguous()


def attn_fwd_sharded(q, k, v, *, world: int, rank: int, scale: Optional[float] = None, causal: bool = True,
                     stream=None):
    """Forward on this rank's heads of the full dense q, k, v [B, H, N, d].
    Returns (o_local, lse_local) for heads head_range(H, world, rank)."""
    from . import attn_fwd
    ql, kl, vl = (local_heads(t, world, rank) for t in (q, k, v))
    if scale is None:
        scale = q.shape[-1] ** -0.5
    if ql.shape[1] == 0:
        return torch.empty_like(ql), torch.empty(ql.shape[:3], device=ql.device, dtype=torch.float32)
    return attn_fwd(ql, kl, vl, scale=scale, causal=causal, stream=stream)


def attn_bwd_sharded(q, k, v, o_local, lse_local, do, *, world: int, rank: int, scale: Optional[float] = None,
                     causal: bool = True, deterministic: bool = False, stream=None):
    """Backward on this rank's heads (o_local / lse_local from attn_fwd_sharded).
    Returns (dq_local, dk_local, dv_local)."""
    from . import attn_bwd
    ql, kl, vl, dol = (local_heads(t, world, rank) for t in (q, k, v, do))
    if scale is None:
        scale = q.shape[-1] ** -0.5
    if ql.shape[1] == 0:
        return torch.empty_like(ql), torch.empty_like(kl), torch.empty_like(vl)
    return attn_bwd(ql, kl, vl, o_local, lse_local, dol, scale=scale, causal=causal, deterministic=deterministic,
                    stream=stream)


def gather_heads(t_local: torch.Tensor, H: int, group=None) -> torch.Tensor:
    """All ranks' head shards [B, H_r, ...] -> the full [B, H, ...] on every rank, in
    head order.  Shards of unequal size are padded to the largest for the collective
    and cut back afterwards."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    sizes = [head_range(H, world, r) for r in range(world)]
    hmax = max(h1 - h0 for h0, h1 in sizes)
    shape = list(t_local.shape)
    pad = torch.zeros([shape[0], hmax] + shape[2:], dtype=t_local.dtype, device=t_local.device)
    pad[:, :t_local.shape[1]] = t_local
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    return torch.cat([p[:, :h1 - h0] for p, (h0, h1) in zip(parts, sizes)], dim=1)


def max_over_ranks(x: float, device=None, group=None) -> float:
    """The largest of every rank's ``x`` (a time: a multi-GPU step is as slow as its
    slowest rank); ``x`` itself when not running distributed."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
