"""Host side of decode with sequences split across GPUs, on the CPU: block
ranges per rank, the rank-local Block Tables, and the all-gather of
attention states over two and three gloo ranks (127.0.0.1).  Each rank's
state is computed by the oracle here; merging the gathered states must give
the oracle's attention over whole sequences."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as O
import workloads as W
from paged_kv_cache_407_b200.binding import state_buffer, state_views
from paged_kv_cache_407_b200.seqsplit import block_range, exchange_states, shard_tables


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_block_ranges_partition_every_sequence():
    for nb in range(0, 40):
        for world in range(1, 9):
            ranges = [block_range(nb, r, world) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == nb
            assert all(ranges[r][1] == ranges[r + 1][0] for r in range(world - 1))
            sizes = [hi - lo for lo, hi in ranges]
            assert max(sizes) - min(sizes) <= 1


def test_local_tables_cover_each_token_once():
    b = W.small_case(41, num_seqs=7, num_q_heads=4, num_kv_heads=2, head_dim=8, block_size=8,
                     dtype=W.F16, max_len=90, lens=[1, 7, 8, 9, 33, 64, 90])
    B = b.block_size
    for world in (1, 2, 3, 4, 16):
        owned = {s: [] for s in range(b.num_seqs)}
        for r in range(world):
            tab, lens = shard_tables(b.block_tables, b.context_lens, B, r, world)
            for s in range(b.num_seqs):
                lo, _ = block_range(-(-int(b.context_lens[s]) // B), r, world)
                for i in range(int(lens[s])):  # local token i is global token lo*B + i
                    assert tab[s, i // B] == b.block_tables[s, lo + i // B]
                    owned[s].append(lo * B + i)
                assert (tab[s, -(-int(lens[s]) // B):] == -1).all()
        for s in range(b.num_seqs):
            assert sorted(owned[s]) == list(range(int(b.context_lens[s]))), (world, s)


def _oracle_state(b, kc, vc, tables, lens):
    """Per (sequence, query head): normalised output and natural log-sum-exp
    over the tokens the tables describe (oracle, float64)."""
    S, Hq, D = b.q.shape
    Hkv = kc.shape[1]
    o = np.zeros((S, Hq, D))
    lse = np.full((S, Hq), -np.inf)
    for s in range(S):
        q = O.decode_bits(b.q[s], b.dtype)
        K = O.decode_bits(O.materialize(kc, tables[s], int(lens[s]), b.block_size), b.dtype)
        V = O.decode_bits(O.materialize(vc, tables[s], int(lens[s]), b.block_size), b.dtype)
        for h in range(Hq):
            g = O.kv_head_of(h, Hq, Hkv)
            m, l, on = O.partial_state(q[h:h + 1], K[g], V[g], b.scale)
            if l[0] > 0:
                o[s, h] = on[0] / l[0]
                lse[s, h] = m[0] + np.log(l[0])
    return o, lse


def _batch():
    return W.small_case(43, num_seqs=5, num_q_heads=8, num_kv_heads=2, head_dim=16, block_size=8,
                        dtype=W.BF16, max_len=200, lens=[3, 17, 64, 150, 200], key_outlier_frac=0.05)


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        b = _batch()
        kc, vc = O.reshape_and_cache(b.k_cache, b.v_cache, b.key, b.value, b.slot_mapping, b.block_size)
        tab, lens = shard_tables(b.block_tables, b.context_lens, b.block_size, rank, world)
        o, lse = _oracle_state(b, kc, vc, tab, lens)
        S, Hq, D = b.q.shape
        state = state_buffer(S * Hq, D, 1, device="cpu")[0]
        so, sl = state_views(state, S, Hq, D)
        so.copy_(torch.from_numpy(o))
        sl.copy_(torch.from_numpy(lse))
        gathered = exchange_states(state)
        q.put((rank, gathered.double().numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gathered_states_merge_to_whole_sequence_attention(world):
    b = _batch()
    kc, vc = O.reshape_and_cache(b.k_cache, b.v_cache, b.key, b.value, b.slot_mapping, b.block_size)
    ref = O.paged_attention_decode(b.q, kc, vc, b.block_tables, b.context_lens, b.block_size, b.scale, b.dtype)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    mp.start_processes(_worker, args=(world, _free_port(), q), nprocs=world, join=True, start_method="spawn")
    res = dict(q.get(timeout=60) for _ in range(world))
    S, Hq, D = b.q.shape
    rows = S * Hq
    for r in range(1, world):
        assert np.array_equal(res[r], res[0]), "every rank must hold the same gathered states"
    g = res[0]
    assert g.shape == (world, rows * (D + 1))
    outs = g[:, : rows * D].reshape(world, rows, D)
    lses = g[:, rows * D:].reshape(world, rows)
    # (o_r, lse_r) is the partial state (m = lse_r, l = 1, o = o_r)
    merged = O.lse_combine(lses, np.ones_like(lses), outs).reshape(S, Hq, D)
    # the states travelled as fp32
    assert np.max(np.abs(merged - ref)) < 1e-5
