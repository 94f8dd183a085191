"""The N > 1 path on CPU: two gloo ranks split the heads of one problem.

Each rank computes its contiguous share of the heads with the fp64 oracle (the
GPU kernels are not available here), the shares are gathered, and the result
must equal the single-process answer; timing aggregation takes the max over
ranks.  This covers the host logic the multi-GPU bench uses: the head split,
the max-over-ranks time and the whole-job throughput.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from exact_attention_132_b200.multi_gpu import aggregate_throughput, max_over_ranks, shard_range


def test_shard_range_covers_every_unit_once():
    for n in (0, 1, 7, 64, 100):
        for world in (1, 2, 3, 8):
            owned = []
            for r in range(world):
                a, b = shard_range(n, r, world)
                assert 0 <= a <= b <= n
                owned += list(range(a, b))
            assert owned == list(range(n))
            sizes = [shard_range(n, r, world)[1] - shard_range(n, r, world)[0] for r in range(world)]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_range(4, 2, 2)


def test_single_process_aggregation_is_identity():
    assert max_over_ranks(3.5) == 3.5
    tf, t = aggregate_throughput(2e12, 10, 1000.0)
    assert t == 1000.0 and abs(tf - 20.0) < 1e-9


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, ret):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        import oracle
        import workloads
        w = workloads.make_small(2, 3, 96, 16, True, seed=21, backward=False)
        q, k, v = workloads.make_bf16_inputs(w)
        heads = [(b, h) for b in range(w.B) for h in range(w.H)]
        a, b = shard_range(len(heads), rank, world)
        mine = heads[a:b]
        o, lse = oracle.attention_fwd_heads(q, k, v, w.sm_scale, True, mine)
        gathered = [None] * world
        dist.all_gather_object(gathered, (mine, o, lse))
        tmax = max_over_ranks(10.0 + rank, dist)
        tf, t = aggregate_throughput(1e12, 4, 100.0 * (rank + 1), dist)
        if rank == 0:
            o_full, l_full = oracle.attention_fwd(q, k, v, w.sm_scale, True)
            ok = True
            seen = []
            for hs, oo, ll in gathered:
                for i, (bb, hh) in enumerate(hs):
                    seen.append((bb, hh))
                    ok &= np.array_equal(oo[i], o_full[bb, hh]) and np.array_equal(ll[i], l_full[bb, hh])
            ret.put((ok, sorted(seen) == sorted(heads), tmax, tf, t))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_split_heads_and_time_by_max():
    ctx = mp.get_context("spawn")
    ret = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, ret)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    ok, complete, tmax, tf, t = ret.get(timeout=5)
    assert ok and complete
    assert tmax == 11.0
    assert t == 200.0 and abs(tf - 1e12 * 4 * 2 / 0.2 / 1e12) < 1e-9
