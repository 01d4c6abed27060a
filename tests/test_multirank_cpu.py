"""Multi-rank host logic on the CPU: world size 2 over gloo (no GPU)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from dit_resolution_packed_b200.sharding import head_range


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_head_range_partitions_heads():
    for heads in (1, 2, 7, 24):
        for world in (1, 2, 3, 8):
            ranges = [head_range(heads, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == heads
            assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
            sizes = [b - a for a, b in ranges]
            assert max(sizes) - min(sizes) <= 1


def _worker(rank, world, port, q, root):
    import sys
    import traceback
    if root not in sys.path:
        sys.path.insert(0, root)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        import workloads
        from dit_resolution_packed_b200.sharding import gather_heads
        import bench
        p = workloads.random_pack([37, 130, 5], heads=5, head_dim=16, seed=3)
        a, b = head_range(5, world, rank)
        sl = lambda t: t[:, a:b].contiguous()
        out, lse = oracle.varlen_attention(sl(p["q"]), sl(p["k"]), sl(p["v"]), p["cu_seqlens"], p["scale"])
        full_out = gather_heads(torch.from_numpy(out), 5)
        full_lse = gather_heads(torch.from_numpy(lse), 5)
        ref_o, ref_l = oracle.varlen_attention(p["q"], p["k"], p["v"], p["cu_seqlens"], p["scale"])
        ok = np.array_equal(full_out.numpy(), ref_o) and np.array_equal(full_lse.numpy(), ref_l)
        # the benchmark's max-over-ranks timing
        mx = bench.allreduce_max(float(rank + 1), world, torch.device("cpu"))
        bench.barrier(world)
        q.put((rank, ok, mx))
    except Exception:
        q.put((rank, traceback.format_exc(), None))
    finally:
        dist.destroy_process_group()


def test_head_sharded_forward_and_max_over_ranks_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q, root)) for r in range(2)]
    for pr in procs:
        pr.start()
    res = [q.get(timeout=120) for _ in procs]
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    for rank, ok, mx in res:
        assert ok is True, f"rank {rank}: {ok}"
        assert mx == 2.0
