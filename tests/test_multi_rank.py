"""The N>1 path of bench.py on CPU: world-size-2 gloo ranks.

Each rank runs its own layer (weak scaling, no data-path collective); the
only cross-rank traffic is the barrier and the max-over-ranks reduction of
the step time.  These tests check that plumbing and the per-rank inputs.
"""
import os
import socket

import numpy as np

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


def _split_worker(rank, world, port, q):
    """One rank of the KV-head split: the oracle's gate, TopK mask and masked
    attention on this rank's head slice of one layer, gathered on rank 0."""
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    import bench
    import oracle
    from long_context_prefill_attngate_b200 import partition
    from long_context_prefill_attngate_b200 import synthetic as syn
    import torch.distributed as dist
    w, r, _ = bench.dist_setup(world)
    try:
        wl = syn.custom("split", 1, 4, 2, 256, 64, number=17, d_gate=64)
        x = syn.make_inputs(wl)                      # every rank draws the same layer
        xs = partition.slice_layer(x, wl.Hq, wl.Hkv, w, r)
        bits = lambda t: syn.bf16_bits(t)
        s = oracle.gate_scores(bits(xs["q"]), bits(xs["k"]), bits(xs["wq"]), bits(xs["wk"]), theta=wl.rope_theta)
        m = oracle.block_mask(s.astype(np.float32), "topk", k_row=oracle.topk_counts(0.5, wl.nb))
        o, lse = oracle.masked_attention(bits(xs["q"]), bits(xs["k"]), bits(xs["v"]), m)
        parts = [None] * w
        dist.all_gather_object(parts, (r, s, m, o, lse))
        if r == 0:
            parts.sort(key=lambda p: p[0])
            # scores and mask are [B, H, nb, nb]; O and LSE come per (b, h, i) unit, head-major for B = 1
            q.put(tuple(np.concatenate([p[i] for p in parts], axis=1 if i <= 2 else 0) for i in range(1, 5)))
    finally:
        dist.destroy_process_group()


def test_kv_head_split_reassembles_single_rank_layer():
    """World size 2 on CPU: each rank computes its KV-head group's slice of a
    layer with the oracle; the slices, concatenated along the head axis, equal
    the single-rank result bit for bit (scores, mask, O and LSE)."""
    import oracle
    from long_context_prefill_attngate_b200 import synthetic as syn
    world = 2
    ctx = mp.get_context("spawn")
    qu = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_split_worker, args=(r, world, port, qu)) for r in range(world)]
    for p in procs:
        p.start()
    got = qu.get(timeout=300)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    wl = syn.custom("split", 1, 4, 2, 256, 64, number=17, d_gate=64)
    x = syn.make_inputs(wl)
    bits = lambda t: syn.bf16_bits(t)
    s = oracle.gate_scores(bits(x["q"]), bits(x["k"]), bits(x["wq"]), bits(x["wk"]), theta=wl.rope_theta)
    m = oracle.block_mask(s.astype(np.float32), "topk", k_row=oracle.topk_counts(0.5, wl.nb))
    o, lse = oracle.masked_attention(bits(x["q"]), bits(x["k"]), bits(x["v"]), m)
    for a, b in zip(got, (s, m, o, lse)):
        assert a.shape == b.shape
        assert np.array_equal(a, b)


def test_head_range_partition():
    from long_context_prefill_attngate_b200 import partition
    assert partition.head_range(32, 8, 4, 1) == (8, 16, 2, 4)
    assert partition.head_range(40, 8, 8, 7) == (35, 40, 7, 8)
    spans = [partition.head_range(32, 8, 2, r) for r in range(2)]
    assert spans == [(0, 16, 0, 4), (16, 32, 4, 8)]
    with pytest.raises(ValueError):
        partition.head_range(32, 8, 3, 0)
    with pytest.raises(ValueError):
        partition.head_range(32, 8, 2, 2)
