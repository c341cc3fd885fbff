"""The N>1 path of bench.py on CPU: world-size-2 gloo ranks.

Each rank runs its own layer (weak scaling, no data-path collective); the
only cross-rank traffic is the barrier and the max-over-ranks reduction of
the step time.  These tests check that plumbing and the per-rank inputs.
"""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    import bench
    from long_context_prefill_attngate_b200 import synthetic as syn
    w, r, _ = bench.dist_setup(world)
    try:
        assert (w, r) == (world, rank)
        t = bench.max_over_ranks(1.5 + rank, w)
        bench.barrier(w)
        wl = syn.custom("mr", 1, 2, 1, 128, 64, number=5)
        x = syn.make_inputs(wl, seed=wl.seed + 1000 * rank)
        q.put((rank, t, float(x["q"].float().sum())))
    finally:
        import torch.distributed as dist
        dist.destroy_process_group()


def test_two_rank_max_and_distinct_layers():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert [r[1] for r in res] == [2.5, 2.5]          # every rank sees the max
    assert res[0][2] != res[1][2]                     # each rank draws its own layer


def test_weak_scaling_value_formula():
    import bench
    flops = bench.attn_flops(1000, 128)
    assert flops == 4.0 * 64 * 64 * 128 * 1000
    # value = world * flops / max_time
    ms = 2.0
    assert abs(2 * flops / (ms * 1e-3) / 1e12 - 2 * 1000 * 4 * 64 * 64 * 128 / 2e-3 / 1e12) < 1e-9


@pytest.mark.parametrize("g", [1, 2, 3, 4, 5, 8])
def test_tile_order_covers_every_query_block_once(g):
    """Host restatement of the kernel's tile enumeration: every (head, query
    block) appears in exactly one tile half (pairs of heads, or block pairs for
    the leftover head of an odd group)."""
    B, Hkv, nb = 2, 3, 7
    Hq = Hkv * g
    lanes = (g + 1) // 2
    seen = {}
    for u in range(nb * B * Hkv * lanes):
        per_group = nb * lanes
        group, rem = divmod(u, per_group)
        level, lane = divmod(rem, lanes)
        kvh, b = group % Hkv, group // Hkv
        i = nb - 1 - level
        if lane < g // 2:
            halves = [(kvh * g + 2 * lane, i), (kvh * g + 2 * lane + 1, i)]
        else:
            if level & 1:
                continue
            h = kvh * g + g - 1
            halves = [(h, i)] + ([(h, i - 1)] if i >= 1 else [])
        for h, ii in halves:
            key = (b, h, ii)
            assert key not in seen
            assert h // g == kvh
            seen[key] = u
    assert len(seen) == B * Hq * nb
