"""Multi-rank host logic on CPU (gloo, world size 2): the split of a batch
across ranks needs no exchange step, and the bench's timing aggregation takes
the slowest rank."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from gated_delta_rule_80_b200.sharding import shard_heads, shard_sequences


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_shard_sequences_covers_batch():
    for B in (0, 1, 5, 64, 129):
        for world in (1, 2, 3, 8):
            parts = [shard_sequences(B, world, r) for r in range(world)]
            assert parts[0][0] == 0 and parts[-1][1] == B
            assert all(a[1] == b[0] for a, b in zip(parts, parts[1:]))
            sizes = [b - a for a, b in parts]
            assert max(sizes) - min(sizes) <= 1


def test_shard_heads_keeps_groups():
    (h0, h1), (v0, v1) = shard_heads(16, 32, 4, 2)
    assert (h0, h1, v0, v1) == (8, 12, 16, 24)
    for hv in range(v0, v1):
        assert h0 <= hv // 2 < h1
    with pytest.raises(ValueError):
        shard_heads(6, 12, 4, 0)


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import sys
        sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
        import bench
        import workloads as W
        from oracle import gdn as O
        # data parallel: each rank decodes its own sequences against its slots
        B, T, H, HV, K, V, slots = 6, 2, 2, 4, 8, 8, 10
        t = W.gdn_tokens(5, B, T, H, HV, K, V, "f32")
        idx = W.slot_indices(5, B, slots)
        pool, _ = W.host_pool(5, idx.tolist(), HV, K, V, "V_FIRST", "f32")
        a, b = shard_sequences(B, world, rank)
        out, writes = O.gdn_decode_slots(*(t[n][a:b] for n in ("q", "k", "v", "a", "b")), t["A_log"],
                                         t["dt_bias"], pool, idx[a:b])
        gathered = [None] * world
        dist.all_gather_object(gathered, (a, b, out, {k: v[0] for k, v in writes.items()}))
        # timing: the job takes the slowest rank
        total, value = bench.aggregate(10.0 + 5.0 * rank, tokens_per_step=64, steps=100, world=world)
        if rank == 0:
            ref_out, ref_writes = O.gdn_decode_slots(t["q"], t["k"], t["v"], t["a"], t["b"], t["A_log"],
                                                     t["dt_bias"], pool, idx)
            ok = True
            for (a_, b_, o, w) in gathered:
                ok &= bool(np.array_equal(o, ref_out[a_:b_]))
                for key, st in w.items():
                    ok &= bool(np.array_equal(st, ref_writes[key][0]))
            n_keys = sum(len(g[3]) for g in gathered)
            q.put((ok, n_keys == len(ref_writes), total, value))
    finally:
        dist.destroy_process_group()


def test_data_parallel_split_needs_no_exchange():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    ok, complete, total, value = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert ok and complete
    assert total == 15.0
    assert value == pytest.approx(2 * 64 * 100 / 0.015)
