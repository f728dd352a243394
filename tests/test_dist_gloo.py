"""The multi-process path on CPU: two gloo ranks (127.0.0.1).

Decode attention shards by sequence with no exchange on the data path: each
rank decodes its own sequences from its own pool.  These tests check that the
shards reproduce the single-process result, that ranks draw distinct seeded
batches, and that the benchmark's cross-rank reduction (max of times, sum of
bytes) agrees on every rank.
"""

import os
import socket

import numpy as np
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as O
import workloads as W


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _init(rank, world, port):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))


def _step_oracle(b):
    kc, vc = O.copy_blocks(b.k_cache, b.v_cache, b.cow_pairs) if b.cow_pairs.size else (b.k_cache, b.v_cache)
    kc, vc = O.reshape_and_cache(kc, vc, b.key, b.value, b.slot_mapping, b.block_size)
    return O.paged_attention_decode(b.q, kc, vc, b.block_tables, b.context_lens, b.block_size, b.scale, b.dtype)


def _shard_worker(rank, world, port, q):
    _init(rank, world, port)
    try:
        glob = W.prefix_share(31, num_seqs=7, prefix_tokens=40, suffix_range=(5, 60), num_q_heads=8,
                              num_kv_heads=2, head_dim=16, block_size=16)
        mine = W.shard_batch(glob, rank, world)
        out = _step_oracle(mine)
        gathered = [None] * world
        dist.all_gather_object(gathered, out)
        if rank == 0:
            q.put(np.concatenate(gathered, axis=0))
    finally:
        dist.destroy_process_group()


def _bench_worker(rank, world, port, q):
    _init(rank, world, port)
    try:
        import bench
        b = bench.build_workload("tiny", rank)
        sig = int(b.q.astype(np.int64).sum())
        sigs = [None] * world
        dist.all_gather_object(sigs, sig)
        (t_max, a_max, e_max), (byts, seqs) = bench.reduce_across_ranks(
            [1.0 + rank, 10.0 * (2 - rank), 3.0], [100.0 * (rank + 1), 4.0], "cpu")
        q.put((rank, sigs, t_max, a_max, e_max, byts, seqs))
    finally:
        dist.destroy_process_group()


def test_sequence_shards_reproduce_the_global_batch():
    glob = W.prefix_share(31, num_seqs=7, prefix_tokens=40, suffix_range=(5, 60), num_q_heads=8,
                          num_kv_heads=2, head_dim=16, block_size=16)
    ref = _step_oracle(glob)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    mp.start_processes(_shard_worker, args=(2, _free_port(), q), nprocs=2, join=True, start_method="spawn")
    got = q.get(timeout=60)
    assert np.array_equal(got, ref)


def test_bench_reduction_and_distinct_rank_batches():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    mp.start_processes(_bench_worker, args=(2, _free_port(), q), nprocs=2, join=True, start_method="spawn")
    res = sorted(q.get(timeout=60) for _ in range(2))
    for rank, sigs, t_max, a_max, e_max, byts, seqs in res:
        assert sigs[0] != sigs[1], "ranks must draw different batches"
        assert (t_max, a_max, e_max) == (2.0, 20.0, 3.0)
        assert (byts, seqs) == (300.0, 8.0)


def test_shard_helper_single_process():
    glob = W.small_case(5, num_seqs=9, num_q_heads=4, num_kv_heads=2, head_dim=8, block_size=8,
                        dtype=W.BF16, max_len=50)
    ref = _step_oracle(glob)
    parts = [_step_oracle(W.shard_batch(glob, r, 3)) for r in range(3)]
    assert np.array_equal(np.concatenate(parts), ref)
    for r in range(3):
        sb = W.shard_batch(glob, r, 3)
        assert sb.num_blocks <= glob.num_blocks and sb.block_tables.max() < sb.num_blocks
