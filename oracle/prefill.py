"""Oracle for paged (chunked) prefill attention: plain, float64, CPU only.

TEST INFRASTRUCTURE ONLY (see ``oracle.paged_kv``).

Sources: lshu.cn/news/11644, vLLM architecture analysis, section
"整体架构" (the scheduler's iteration: a new request's prompt is prefilled,
a long prompt in several chunks over several iterations) and section
"性能关键路径与瓶颈" (prefill is compute-bound on the tensor cores; chunked
prefill spreads one long prompt over iterations).  Attention itself is the
textbook softmax attention; causality (a token sees the tokens up to and
including itself) is the defining property of generating left to right.

Reading (the pages print no formula): one prefill call serves, for each
sequence s, a chunk of C_s new tokens that are the last C_s of its L_s
tokens; their K/V are already in the cache (written by the cache write of
the same iteration, as in decode).  The token at position p (L_s - C_s <= p
< L_s) attends over positions 0 .. p of its own sequence.  C_s = 1 is a
decode step; C_s = L_s is the prefill of a whole prompt.
"""

from __future__ import annotations

import numpy as np

from .paged_kv import attend, decode_bits, kv_head_of, materialize


def paged_prefill(q_bits, k_cache, v_cache, block_tables, query_start, context_lens, block_size, scale, dtype,
                  seqs=None) -> np.ndarray:
    """``q_bits [T, Hq, D]``: the chunks' queries, sequence s owning rows
    ``query_start[s] .. query_start[s+1]``; caches ``[N, Hkv, B, D]`` (bits);
    ``block_tables [S, max_blocks]``; ``context_lens [S]`` (L_s, chunk
    included).  Returns float64 ``[T, Hq, D]`` (rows of unlisted sequences
    NaN)."""
    T, Hq, D = q_bits.shape
    Hkv = k_cache.shape[1]
    out = np.full((T, Hq, D), np.nan)
    S = len(context_lens)
    for s in (range(S) if seqs is None else seqs):
        t0, t1 = int(query_start[s]), int(query_start[s + 1])
        C, L = t1 - t0, int(context_lens[s])
        if C == 0:
            continue
        K = decode_bits(materialize(k_cache, block_tables[s], L, block_size), dtype)  # [Hkv, L, D]
        V = decode_bits(materialize(v_cache, block_tables[s], L, block_size), dtype)
        for j in range(C):
            p = L - C + j  # position of the chunk's j-th token
            q = decode_bits(q_bits[t0 + j], dtype)
            for g in range(Hkv):
                heads = [h for h in range(Hq) if kv_head_of(h, Hq, Hkv) == g]
                out[t0 + j, heads] = attend(q[heads], K[g, : p + 1], V[g, : p + 1], scale)
    return out
