"""Multi-GPU plumbing: one process per GPU over torch.distributed.

Every (batch, head, query block) of the forward pass is independent, so the
path shards with no exchange inside it:

* ``bench.py --gpus N`` runs one independent problem per GPU (weak scaling) and
  only reduces the timings (max over ranks);
* ``fwd_sharded`` splits the B*H heads of ONE problem into contiguous per-rank
  ranges, runs the CUDA forward on the local range and, if asked, all-gathers
  O and LSE so every rank holds the full result.

Nothing here does attention arithmetic; the local compute is the C-ABI call.
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def rank_env() -> tuple[int, int, int]:
    """(rank, world_size, local_rank) from the torchrun environment (0, 1, 0 alone)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str, timeout_s: float = 120.0, device: torch.device | None = None) -> None:
    """Initialise the default process group from the environment (torchrun sets
    MASTER_ADDR/PORT, RANK, WORLD_SIZE) with a short timeout, so ranks waiting
    on a missing peer fail instead of hanging."""
    if dist.is_initialized():
        return
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
    if device is not None and backend == "nccl":
        kw["device_id"] = device
    dist.init_process_group(backend, **kw)


def max_over_ranks(values, device) -> list[float]:
    """Element-wise max of a list of floats over all ranks (identity alone)."""
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def shard_plan(n_units: int, world: int) -> list[tuple[int, int]]:
    """Contiguous [start, end) ranges covering n_units, one per rank, sizes
    differing by at most one (earlier ranks take the extra unit)."""
    if world <= 0:
        raise ValueError("world must be positive")
    base, extra = divmod(n_units, world)
    out, s = [], 0
    for r in range(world):
        e = s + base + (1 if r < extra else 0)
        out.append((s, e))
        s = e
    return out


def gather_heads(local: torch.Tensor, plan, n_units: int, group=None) -> torch.Tensor:
    """All-gather per-rank slices along dim 0 (the flattened B*H axis) into the
    full [n_units, ...] tensor on every rank.  Ranks may own unequal counts."""
    world = len(plan)
    if world == 1:
        return local
    width = max(e - s for s, e in plan)
    tail = tuple(local.shape[1:])
    padded = torch.zeros((width,) + tail, dtype=local.dtype, device=local.device)
    padded[: local.shape[0]] = local
    parts = [torch.empty_like(padded) for _ in range(world)]
    dist.all_gather(parts, padded, group=group)
    full = torch.empty((n_units,) + tail, dtype=local.dtype, device=local.device)
    for (s, e), p in zip(plan, parts):
        full[s:e] = p[: e - s]
    return full


def fwd_sharded(q, k, v, causal: bool = False, scale: float | None = None, gather: bool = True):
    """Forward attention of one [B,H,N,d] problem split over the ranks by heads.

    Each rank computes its contiguous range of the B*H heads with the CUDA
    kernel (``binding.fwd``); with ``gather`` every rank receives the full O
    [B,H,Nq,d] and LSE [B,H,Nq], otherwise each rank returns (o_local,
    lse_local, (start, end)) for its range of the flattened B*H axis.
    """
    from . import binding

    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    world = dist.get_world_size() if dist.is_initialized() else 1
    rank = dist.get_rank() if dist.is_initialized() else 0
    plan = shard_plan(B * H, world)
    s, e = plan[rank]
    q2 = q.reshape(B * H, 1, Nq, d)[s:e].reshape(1, e - s, Nq, d)
    k2 = k.reshape(B * H, 1, Nk, d)[s:e].reshape(1, e - s, Nk, d)
    v2 = v.reshape(B * H, 1, Nk, d)[s:e].reshape(1, e - s, Nk, d)
    if e > s:
        o2, l2 = binding.fwd(q2.contiguous(), k2.contiguous(), v2.contiguous(), causal=causal,
                             scale=scale)
        o2 = o2.reshape(e - s, Nq, d)
        l2 = l2.reshape(e - s, Nq)
    else:
        o2 = torch.empty((0, Nq, d), dtype=q.dtype, device=q.device)
        l2 = torch.empty((0, Nq), dtype=torch.float32, device=q.device)
    if not gather:
        return o2, l2, (s, e)
    o = gather_heads(o2, plan, B * H).reshape(B, H, Nq, d)
    lse = gather_heads(l2, plan, B * H).reshape(B, H, Nq)
    return o, lse
