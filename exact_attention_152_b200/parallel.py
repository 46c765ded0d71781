"""Multi-GPU plumbing: one process per GPU over torch.distributed.

Every (batch, head, query block) of the forward pass is independent, so the
path shards with no exchange inside it:

* ``bench.py --gpus N`` runs one independent problem per GPU (weak scaling) and
  only reduces the timings (max over ranks);
* ``fwd_sharded`` splits ONE problem by key/value-head groups: a rank owns
  whole groups -- one key/value head with the H/Hkv query heads that read it
  (grouped-query attention; H/Hkv = 1 for multi-head attention) -- so it needs
  only its own K/V heads.  It runs the CUDA forward on that range and, if
  asked, all-gathers O and LSE so every rank holds the full result.

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


def group_plan(B: int, H: int, Hkv: int, world: int):
    """Per-rank ranges for a problem of B*H query heads over B*Hkv key/value
    heads: the key/value heads are split into contiguous ranges (shard_plan),
    and a rank's query heads are those of its key/value heads.  Query head h
    of batch entry b reads key/value head h // (H // Hkv), so in the flattened
    B*H axis the query heads of key/value heads [s, e) are [s*G, e*G) with
    G = H // Hkv.  Returns (kv_plan, q_plan)."""
    if Hkv <= 0 or H % Hkv != 0:
        raise ValueError("H must be a positive multiple of Hkv")
    G = H // Hkv
    kv_plan = shard_plan(B * Hkv, world)
    q_plan = [(s * G, e * G) for s, e in kv_plan]
    return kv_plan, q_plan


def fwd_sharded(q, k, v, causal: bool = False, scale: float | None = None, gather: bool = True,
                window=None):
    """Forward attention of one problem, q [B,H,Nq,d] and k/v [B,Hkv,Nk,d]
    (Hkv divides H), split over the ranks by key/value-head groups.

    Each rank computes the query heads of its contiguous range of key/value
    heads with the CUDA kernel (``binding.fwd``: attn_fwd, attn_fwd_gqa or
    attn_fwd_window); every load stays in the rank's own memory.  With
    ``gather`` every rank receives the full O [B,H,Nq,d] and LSE [B,H,Nq]
    (one NCCL all-gather each); otherwise each rank returns (o_local,
    lse_local, (start, end)) for its range of the flattened B*H axis.
    """
    from . import binding

    B, H, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    world = dist.get_world_size() if dist.is_initialized() else 1
    rank = dist.get_rank() if dist.is_initialized() else 0
    kv_plan, q_plan = group_plan(B, H, Hkv, world)
    ks, ke = kv_plan[rank]
    s, e = q_plan[rank]
    if e > s:
        q2 = q.reshape(B * H, Nq, d)[s:e].reshape(1, e - s, Nq, d).contiguous()
        k2 = k.reshape(B * Hkv, Nk, d)[ks:ke].reshape(1, ke - ks, Nk, d).contiguous()
        v2 = v.reshape(B * Hkv, Nk, d)[ks:ke].reshape(1, ke - ks, Nk, d).contiguous()
        o2, l2 = binding.fwd(q2, k2, v2, causal=causal, scale=scale, window=window)
        o2 = o2.reshape(e - s, Nq, d)
        l2 = l2.reshape(e - s, Nq)
    else:
        o2 = torch.empty((0, Nq, d), dtype=q.dtype, device=q.device)
        l2 = torch.empty((0, Nq), dtype=torch.float32, device=q.device)
    if not gather:
        return o2, l2, (s, e)
    o = gather_heads(o2, q_plan, B * H).reshape(B, H, Nq, d)
    lse = gather_heads(l2, q_plan, B * H).reshape(B, H, Nq)
    return o, lse
