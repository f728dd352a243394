"""Decode of long sequences split across GPUs: each rank holds a contiguous
range of every sequence's blocks, computes an attention state (normalised
fp32 output + log-sum-exp) over its tokens, the ranks all-gather the states,
and every rank merges them into the output.

The exchange is one all-gather of ``S * Hq * (D + 1)`` fp32 per rank (66 KB
for 4 sequences x 32 heads x 128 dims), the only collective of the split
path.  Merging states over disjoint token sets is the split-K identity of
softmax attention (with w_r = exp(lse_r - max lse): out = sum w_r o_r / sum
w_r).  The compute steps are the library calls
``paged_attention_decode_lse`` and ``merge_attention_states``; this module
holds the host side: which blocks each rank owns, the state buffer, and the
collective.
"""

from __future__ import annotations

import numpy as np
import torch
import torch.distributed as dist

from .binding import merge_attention_states, paged_attention_decode_lse, state_buffer, state_views


def block_range(num_blocks: int, rank: int, world: int) -> tuple[int, int]:
    """Logical blocks [lo, hi) of a sequence of ``num_blocks`` blocks that
    ``rank`` of ``world`` owns: contiguous, sizes differing by at most one,
    lower ranks first."""
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    return rank * num_blocks // world, (rank + 1) * num_blocks // world


def shard_tables(block_tables: np.ndarray, context_lens: np.ndarray, block_size: int, rank: int,
                 world: int) -> tuple[np.ndarray, np.ndarray]:
    """The rank's Block Table rows (its range of each sequence, padded with
    -1) and its token counts.  Token i of sequence s belongs to the rank that
    owns logical block i // block_size; every token has exactly one owner."""
    tables = np.asarray(block_tables, dtype=np.int32)
    lens = np.asarray(context_lens, dtype=np.int64)
    S = tables.shape[0]
    nbs = -(-lens // block_size)
    ranges = [block_range(int(nb), rank, world) for nb in nbs]
    width = max([1] + [hi - lo for lo, hi in ranges])
    local = np.full((S, width), -1, dtype=np.int32)
    local_lens = np.zeros(S, dtype=np.int32)
    for s, (lo, hi) in enumerate(ranges):
        local[s, : hi - lo] = tables[s, lo:hi]
        local_lens[s] = max(0, min(int(lens[s]), hi * block_size) - lo * block_size)
    return local, local_lens


def exchange_states(state: torch.Tensor, group=None) -> torch.Tensor:
    """All-gather one rank's flat fp32 state into ``[world, numel]``."""
    world = dist.get_world_size(group)
    out = torch.empty(world * state.numel(), dtype=state.dtype, device=state.device)
    dist.all_gather_into_tensor(out, state.contiguous().view(-1), group=group)
    return out.view(world, state.numel())


def split_decode(out, query, k_cache, v_cache, local_tables, local_lens, max_local_len, scale, group=None,
                 partition_size=0, workspace=None, d_status=None):
    """One decode call of sequences split across the ranks of ``group``:
    ``local_tables`` / ``local_lens`` (device int32) describe this rank's
    share (``shard_tables``); ``out`` receives the full attention on every
    rank.  Returns the gathered states ``[world, rows * (D + 1)]``."""
    S, Hq, D = query.shape
    state = state_buffer(S * Hq, D, 1, device=query.device)[0]
    o, lse = state_views(state, S, Hq, D)
    paged_attention_decode_lse(o, lse, query, k_cache, v_cache, local_tables, local_lens, max_local_len, scale,
                               partition_size=partition_size, workspace=workspace, d_status=d_status)
    gathered = exchange_states(state, group)
    merge_attention_states(out, gathered)
    return gathered
