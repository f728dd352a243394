"""Algorithmic byte counts of the hot-path calls (host arithmetic only).

These are the bytes a call must move at minimum, used for GB/s and roofline
fractions: every byte counted once, K/V at their exact token counts (the tail
of a partially filled block is not counted), no re-reads, no workspace.
"""

from __future__ import annotations

import numpy as np


def decode_bytes(context_lens, num_q_heads: int, num_kv_heads: int, head_dim: int,
                 block_size: int, elem_bytes: int = 2, kv_elem_bytes: int | None = None) -> dict:
    """Bytes of one decode-attention call: K and V of every context token,
    the queries, the outputs, the Block Table entries in use and the lengths.
    ``kv_elem_bytes``: bytes per cached K/V element (1 for 8-bit pools;
    default ``elem_bytes``)."""
    lens = np.asarray(context_lens, dtype=np.int64)
    S = lens.size
    kv_b = elem_bytes if kv_elem_bytes is None else kv_elem_bytes
    kv = int(lens.sum()) * num_kv_heads * head_dim * kv_b * 2
    q = S * num_q_heads * head_dim * elem_bytes
    out = q
    tables = int(((lens + block_size - 1) // block_size).sum()) * 4
    return {"kv": kv, "q": q, "out": out, "tables": tables, "lens": 4 * S,
            "total": kv + q + out + tables + 4 * S}


def decode_bytes_padded_kv(context_lens, num_kv_heads: int, head_dim: int, block_size: int,
                           elem_bytes: int = 2) -> int:
    """K+V bytes when every used block is counted whole (what a block-granular
    reader may fetch)."""
    lens = np.asarray(context_lens, dtype=np.int64)
    nb = (lens + block_size - 1) // block_size
    return int(nb.sum()) * block_size * num_kv_heads * head_dim * elem_bytes * 2


def unique_kv_bytes(block_tables, context_lens, num_kv_heads: int, head_dim: int, block_size: int,
                    elem_bytes: int = 2) -> int:
    """K+V bytes of the distinct physical blocks a call reads, each at the
    largest number of its tokens any sequence uses (a block shared by several
    sequences' tables counts once)."""
    tables = np.asarray(block_tables)
    lens = np.asarray(context_lens, dtype=np.int64)
    used = {}
    for s, L in enumerate(lens):
        nb = (int(L) + block_size - 1) // block_size
        for j in range(nb):
            blk = int(tables[s, j])
            used[blk] = max(used.get(blk, 0), min(block_size, int(L) - j * block_size))
    return sum(used.values()) * num_kv_heads * head_dim * elem_bytes * 2


def split_partials_bytes(context_lens, num_q_heads: int, head_dim: int, partition_tokens: int) -> int:
    """Workspace traffic of split-K (implementation overhead, not algorithmic):
    every sequence that spans more than one partition writes one fp32 (m, l,
    o[D]) state per (query head, partition) and its merge reads each back."""
    lens = np.asarray(context_lens, dtype=np.int64)
    parts = (lens + partition_tokens - 1) // partition_tokens
    states = int(parts[parts > 1].sum()) * num_q_heads
    return states * (head_dim + 2) * 4 * 2


def reshape_and_cache_bytes(num_tokens: int, num_kv_heads: int, head_dim: int,
                            elem_bytes: int = 2, cache_elem_bytes: int | None = None) -> int:
    """Read the new K and V rows, write them into the pool, read the slots."""
    c_b = elem_bytes if cache_elem_bytes is None else cache_elem_bytes
    rows = num_tokens * num_kv_heads * head_dim * 2
    return rows * elem_bytes + rows * c_b + 8 * num_tokens


def copy_blocks_bytes(num_pairs: int, num_kv_heads: int, block_size: int, head_dim: int,
                      elem_bytes: int = 2) -> int:
    """Read and write one whole block of each pool per pair, plus the pairs."""
    block = num_kv_heads * block_size * head_dim * elem_bytes
    return num_pairs * (2 * 2 * block + 16)


def kv_bytes_per_token(num_layers: int, hidden: int, elem_bytes: int = 2) -> int:
    """KV-cache bytes one token occupies across a model: K and V of every layer."""
    return 2 * num_layers * hidden * elem_bytes


def static_reservation_waste(reserved_slots: int, used_slots: int) -> float:
    """Fraction of a statically reserved KV region that stays unused."""
    return 1.0 - used_slots / reserved_slots


def block_fragmentation(context_lens, block_size: int) -> float:
    """Fraction of allocated block slots that hold no token (internal
    fragmentation of the last block of every sequence)."""
    lens = np.asarray(context_lens, dtype=np.int64)
    alloc = ((lens + block_size - 1) // block_size) * block_size
    return float((alloc - lens).sum() / alloc.sum())


def prefill_flops(context_lens, chunk_lens, num_q_heads: int, head_dim: int) -> float:
    """Algorithmic FLOPs of a causal prefill call: the chunk's token at
    position p attends over p + 1 keys, 2 D FLOPs each for Q K^T and for P V,
    per query head."""
    total = 0
    for L, C in zip(np.asarray(context_lens).tolist(), np.asarray(chunk_lens).tolist()):
        # sum over p = L - C .. L - 1 of (p + 1)
        total += (L * (L + 1) - (L - C) * (L - C + 1)) // 2
    return float(4 * head_dim * num_q_heads * total)


def prefill_bytes(context_lens, chunk_lens, num_q_heads: int, num_kv_heads: int, head_dim: int,
                  elem_bytes: int = 2) -> int:
    """Bytes a prefill call must move at least once: every context token's K
    and V, the chunk's queries and outputs."""
    kv = int(np.sum(context_lens)) * num_kv_heads * head_dim * elem_bytes * 2
    qo = int(np.sum(chunk_lens)) * num_q_heads * head_dim * elem_bytes * 2
    return kv + qo
