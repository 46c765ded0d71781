"""Multi-process plumbing on CPU (gloo, world size 2) and the sharded forward on
one GPU.  The forward pass has no data-path collective; these cover the rank
environment, the max-over-ranks timing reduction, the head sharding plan and
the all-gather that assembles a sharded result."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from exact_attention_152_b200 import parallel


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_shard_plan_covers_every_unit_once():
    for n in (0, 1, 7, 32, 33, 1000):
        for world in (1, 2, 3, 8):
            plan = parallel.shard_plan(n, world)
            assert len(plan) == world and plan[0][0] == 0 and plan[-1][1] == n
            assert all(plan[i][1] == plan[i + 1][0] for i in range(world - 1))
            sizes = [e - s for s, e in plan]
            assert max(sizes) - min(sizes) <= 1


def test_group_plan_keeps_groups_whole():
    """Every query head lands on the rank that owns the key/value head it
    reads, each exactly once, for MHA, GQA and MQA shapes."""
    for B, H, Hkv in ((1, 1, 1), (2, 32, 8), (3, 6, 2), (2, 8, 1), (1, 16, 16), (2, 4, 4)):
        G = H // Hkv
        for world in (1, 2, 3, 4, 8):
            kv_plan, q_plan = parallel.group_plan(B, H, Hkv, world)
            owner = {}
            for r, ((ks, ke), (s, e)) in enumerate(zip(kv_plan, q_plan)):
                assert (e - s) == (ke - ks) * G
                for flat in range(s, e):
                    b, h = divmod(flat, H)
                    assert ks <= b * Hkv + h // G < ke, (B, H, Hkv, world, r, flat)
                    assert flat not in owner
                    owner[flat] = r
            assert sorted(owner) == list(range(B * H))
    with pytest.raises(ValueError):
        parallel.group_plan(1, 6, 4, 2)


def _worker(rank, world, port, q):
    try:
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                          WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
        assert parallel.rank_env() == (rank, world, rank)
        parallel.init("gloo", timeout_s=60)
        # timing reduction: max over ranks, element-wise
        m = parallel.max_over_ranks([1.0 + rank, 10.0 - rank], torch.device("cpu"))
        assert m == [float(world), 10.0], m
        # sharded result assembly with unequal shards (5 heads over 2 ranks)
        n, nq, d = 5, 3, 4
        plan = parallel.shard_plan(n, world)
        s, e = plan[rank]
        local = torch.arange(s, e, dtype=torch.float32)[:, None, None].expand(e - s, nq, d).contiguous()
        full = parallel.gather_heads(local, plan, n)
        want = torch.arange(n, dtype=torch.float32)[:, None, None].expand(n, nq, d)
        assert torch.equal(full, want)
        lse_local = torch.full((e - s, nq), float(rank))
        lse_full = parallel.gather_heads(lse_local, plan, n)
        assert torch.equal(lse_full[:3], torch.zeros(3, nq)) and torch.equal(lse_full[3:], torch.ones(2, nq))
        # grouped-query plan (B=2, H=6, Hkv=3 -> 6 key/value heads, 2 query heads
        # each): each rank assembles the query heads of its own key/value heads,
        # tagged with the key/value head they read; the gather restores the order
        B, H, Hkv = 2, 6, 3
        G = H // Hkv
        kv_plan, q_plan = parallel.group_plan(B, H, Hkv, world)
        (ks, ke), (s, e) = kv_plan[rank], q_plan[rank]
        kv_of = torch.arange(ks, ke, dtype=torch.float32).repeat_interleave(G)
        local = kv_of[:, None, None].expand(e - s, nq, d).contiguous()
        full = parallel.gather_heads(local, q_plan, B * H)
        flat = torch.arange(B * H)
        want = ((flat // H) * Hkv + (flat % H) // G).float()[:, None, None].expand(B * H, nq, d)
        assert torch.equal(full, want)
        dist.barrier()
        dist.destroy_process_group()
        q.put((rank, "ok"))
    except Exception as exc:  # report to the parent instead of hanging it
        q.put((rank, repr(exc)))


def test_gloo_world_size_two():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert results == {0: "ok", 1: "ok"}, results


@pytest.mark.gpu
def test_fwd_sharded_single_rank_matches_fwd():
    from exact_attention_152_b200 import binding
    g = torch.Generator().manual_seed(3)
    q, k, v = (torch.randn(2, 3, 200, 64, generator=g).to(torch.bfloat16).cuda() for _ in range(3))
    o, lse = parallel.fwd_sharded(q, k, v, causal=True)
    o_ref, lse_ref = binding.fwd(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o.view(torch.int16), o_ref.view(torch.int16))
    assert torch.equal(lse, lse_ref)
    o2, l2, (s, e) = parallel.fwd_sharded(q, k, v, causal=True, gather=False)
    assert (s, e) == (0, 6) and torch.equal(o2.view(torch.int16), o_ref.reshape(6, 200, 64).view(torch.int16))


@pytest.mark.gpu
@pytest.mark.parametrize("Hkv,window", [(2, None), (1, None), (4, (63, 0))])
def test_fwd_sharded_gqa_matches_fwd(Hkv, window):
    """A grouped-query problem through the sharded path equals attn_fwd_gqa (or
    attn_fwd_window) bit for bit, and a rank's local slice of a simulated
    2-rank plan equals the same heads of the full result."""
    from exact_attention_152_b200 import binding
    g = torch.Generator().manual_seed(4)
    B, H, N, d = 2, 8, 300, 128
    q = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16).cuda()
    k, v = (torch.randn(B, Hkv, N, d, generator=g).to(torch.bfloat16).cuda() for _ in range(2))
    causal = window is None
    o, lse = parallel.fwd_sharded(q, k, v, causal=causal, window=window)
    o_ref, lse_ref = binding.fwd(q, k, v, causal=causal, window=window)
    torch.cuda.synchronize()
    assert torch.equal(o.view(torch.int16), o_ref.view(torch.int16))
    assert torch.equal(lse, lse_ref)
    # rank 1 of 2: its key/value heads and their query heads, computed alone
    kv_plan, q_plan = parallel.group_plan(B, H, Hkv, 2)
    (ks, ke), (s, e) = kv_plan[1], q_plan[1]
    q2 = q.reshape(B * H, N, d)[s:e].reshape(1, e - s, N, d).contiguous()
    k2 = k.reshape(B * Hkv, N, d)[ks:ke].reshape(1, ke - ks, N, d).contiguous()
    v2 = v.reshape(B * Hkv, N, d)[ks:ke].reshape(1, ke - ks, N, d).contiguous()
    o2, _ = binding.fwd(q2, k2, v2, causal=causal, window=window)
    torch.cuda.synchronize()
    assert torch.equal(o2.reshape(e - s, N, d).view(torch.int16),
                       o_ref.reshape(B * H, N, d)[s:e].view(torch.int16))
