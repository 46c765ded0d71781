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
