"""Byte accounting against the closed forms the pages print (CPU)."""

import numpy as np

from paged_kv_cache_407_b200 import accounting as A


def test_kv_bytes_per_token_7b():
    """lshu.cn/news/11644, "问题：KV Cache 的内存困境": a 7B model produces about
    0.5 MB of fp16 KV cache per token (32 layers, hidden size 4096)."""
    assert A.kv_bytes_per_token(32, 4096, 2) == 512 * 1024


def test_static_reservation_waste():
    """Same section: 2048 reserved slots of which requests use 256 on average
    leave about 87% of the KV cache idle."""
    assert abs(A.static_reservation_waste(2048, 256) - 0.875) < 1e-12


def test_decode_bytes_small():
    lens = [1, 15, 16, 33]
    b = A.decode_bytes(lens, num_q_heads=4, num_kv_heads=4, head_dim=64, block_size=16)
    assert b["kv"] == 65 * 4 * 64 * 2 * 2
    assert b["q"] == b["out"] == 4 * 4 * 64 * 2
    assert b["tables"] == (1 + 1 + 1 + 3) * 4
    assert b["total"] == b["kv"] + 2 * b["q"] + b["tables"] + 16
    assert A.decode_bytes_padded_kv(lens, 4, 64, 16) == 6 * 16 * 4 * 64 * 4


def test_fragmentation_under_one_block_per_sequence():
    """Paging wastes at most the unused tail of each sequence's last block
    (ypxx.net, "2.1 PagedAttention分页注意力核心机制": waste under 4%)."""
    rng = np.random.default_rng(0)
    lens = rng.integers(128, 2049, size=64)
    f = A.block_fragmentation(lens, 16)
    assert 0 < f < 0.04
    assert A.block_fragmentation([16, 32], 16) == 0.0
    assert abs(A.block_fragmentation([1], 16) - 15 / 16) < 1e-12


def test_copy_and_write_bytes():
    assert A.copy_blocks_bytes(128, 8, 16, 128) == 128 * (4 * 8 * 16 * 128 * 2 + 16)
    assert A.reshape_and_cache_bytes(256, 8, 128) == 2 * 256 * 8 * 128 * 2 * 2 + 8 * 256


def test_prefill_flops_is_the_causal_count():
    """Brute force: the chunk token at position p attends over p + 1 keys;
    Q K^T and P V are 2 D FLOPs per (key, query head) each."""
    from paged_kv_cache_407_b200 import accounting as A
    lens, chunks, Hq, D = [10, 7, 300, 1], [10, 3, 17, 1], 6, 64
    brute = 0
    for L, C in zip(lens, chunks):
        for p in range(L - C, L):
            brute += Hq * (2 * D * (p + 1) + 2 * D * (p + 1))
    assert A.prefill_flops(lens, chunks, Hq, D) == brute
    assert A.prefill_flops([4096] * 4, [4096] * 4, 32, 128) == 4 * 4 * 128 * 32 * 4096 * 4097 // 2
    assert A.prefill_bytes([100], [20], 8, 2, 64) == 100 * 2 * 64 * 2 * 2 + 20 * 8 * 64 * 2 * 2


def test_unique_kv_bytes_counts_a_shared_block_once():
    """Two sequences whose tables share their first two blocks: the shared
    blocks count once, each at the most tokens any sequence uses in it; with
    disjoint tables the unique count equals the logical one."""
    Hkv, D, B = 2, 8, 4
    per_token = Hkv * D * 2 * 2
    tables = np.array([[5, 6, 7, -1], [5, 6, 9, 3]])
    lens = [10, 13]  # seq 0: 4 + 4 + 2 tokens; seq 1: 4 + 4 + 4 + 1
    assert A.unique_kv_bytes(tables, lens, Hkv, D, B) == (4 + 4 + 2 + 4 + 1) * per_token
    disjoint = np.array([[1, 2, 3, -1], [4, 5, 6, 7]])
    logical = A.decode_bytes(lens, 4, Hkv, D, B)["kv"]
    assert A.unique_kv_bytes(disjoint, lens, Hkv, D, B) == logical
    # a block shared where one sequence fills it and the other uses its head
    assert A.unique_kv_bytes(np.array([[0, -1], [0, 1]]), [2, 6], Hkv, D, B) == (4 + 2) * per_token


def test_bench_decode_accounting_on_the_workloads():
    """The bench's side figures on the prefix workload: the shared 1024-token
    prefix counts once in the unique bytes; with private tables (7B batch)
    unique equals logical."""
    import bench
    import workloads as W

    b = W.WORKLOADS["prefix_share"]()
    acc = bench.decode_accounting(b, 2, 1.0)
    per_token = b.num_kv_heads * b.head_dim * 2 * 2
    suffix = int(np.sum(np.asarray(b.context_lens) - 1024))
    # prefix blocks 0..62 shared by every table; block 63 copied per sequence
    assert acc["kv_bytes_unique_blocks"] == (63 * 16 + len(b.context_lens) * 16 + suffix) * per_token
    assert acc["kv_bytes_logical"] == int(np.sum(b.context_lens)) * per_token
    b7 = W.WORKLOADS["tiny"]()
    acc7 = bench.decode_accounting(b7, 2, 1.0)
    assert acc7["kv_bytes_unique_blocks"] == acc7["kv_bytes_logical"]
    assert acc7["kv_bytes_padded_to_blocks"] >= acc7["kv_bytes_logical"]


def test_split_partials_bytes():
    """Only sequences spanning several partitions write and read states:
    lengths 100, 600, 1025 at P = 512 -> 0 + 2 + 3 states per query head."""
    assert A.split_partials_bytes([100, 600, 1025], 4, 128, 512) == (2 + 3) * 4 * 130 * 4 * 2
    assert A.split_partials_bytes([512, 1], 8, 64, 512) == 0
    import types

    import bench

    long_ctx = types.SimpleNamespace(context_lens=[131072] * 4, num_q_heads=32, head_dim=128)
    assert bench.split_partials_bytes(long_ctx, 512) == 4 * 256 * 32 * 130 * 4 * 2  # 34 MB per call
