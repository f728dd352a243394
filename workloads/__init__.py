"""Seeded synthetic paged-KV decode batches.

This module is the one piece shared by the CUDA path's tests and benchmark and
by the oracle's tests.  It only builds inputs: it draws the random values,
places each sequence's tokens into blocks of a shuffled block pool, encodes the
per-token cache slots and the copy-on-write pairs.  It contains no attention
arithmetic and imports neither the oracle nor the CUDA package.

Storage convention (the input format both sides read):

* fp16 / bf16 tensors are carried as ``uint16`` arrays of bit patterns, so both
  sides see identical bits and bit-exact comparisons are plain integer
  comparisons.
* ``k_cache`` / ``v_cache``: ``[num_blocks, num_kv_heads, block_size, head_dim]``
  (one contiguous ``block_size x head_dim`` tile per (block, kv head)).
* ``block_tables``: ``int32 [num_seqs, max_blocks]``, padded with -1.
* ``slot_mapping``: ``int64 [num_tokens]``; the slot of a token is
  ``block_id * block_size + offset_in_block``; a negative slot marks padding.
* ``context_lens`` counts every token attended to, including the token written
  in the same step (it is the last position, ``context_len - 1``).

Random-stream order for every batch (so a seed fully fixes the bits):
context lengths (drawn by the workload function), then the pool permutation,
then per sequence in order K ``[L, Hkv, D]`` and V ``[L, Hkv, D]`` (float32
standard normal) and, when outliers are requested, one uniform per
(token, kv head); the queries ``[S, Hq, D]`` are drawn last.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

F16 = "f16"
BF16 = "bf16"
DTYPES = (F16, BF16)

# Quiet-NaN bit patterns with a recognisable payload.  Every slot of the pool
# that no sequence owns (free blocks, the tail of a sequence's last block, and
# the slot a new token is about to be written to) holds this value, so a kernel
# that reads a slot it should not read turns the output into NaN.
POISON_BITS = {F16: 0x7E5A, BF16: 0x7FDA}


def to_bits(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float32 values to fp16/bf16 (round to nearest even), return bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == F16:
        return x.astype(np.float16).view(np.uint16)
    if dtype == BF16:
        u = x.view(np.uint32)
        rounded = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
        return rounded.astype(np.uint16)
    raise ValueError(f"unknown dtype {dtype!r}")


@dataclass
class PagedBatch:
    """One decode step's inputs for one attention layer."""

    name: str
    dtype: str
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    scale: float
    q: np.ndarray  # uint16 [S, Hq, D]
    k_cache: np.ndarray  # uint16 [N, Hkv, B, D]
    v_cache: np.ndarray  # uint16 [N, Hkv, B, D]
    block_tables: np.ndarray  # int32 [S, max_blocks]
    context_lens: np.ndarray  # int32 [S]
    key: np.ndarray  # uint16 [T, Hkv, D]   new tokens' keys
    value: np.ndarray  # uint16 [T, Hkv, D]  new tokens' values
    slot_mapping: np.ndarray  # int64 [T]
    cow_pairs: np.ndarray = field(default_factory=lambda: np.zeros((0, 2), np.int64))
    # Block tables as they were before the copy-on-write pairs were applied
    # (only set when the batch shares blocks between sequences).
    block_tables_before_cow: np.ndarray | None = None
    partition_size: int = 0  # 0 = let the library choose
    seed: int = 0

    @property
    def num_seqs(self) -> int:
        return int(self.context_lens.shape[0])

    @property
    def num_blocks(self) -> int:
        return int(self.k_cache.shape[0])

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max()) if self.num_seqs else 0

    @property
    def num_tokens(self) -> int:
        return int(self.slot_mapping.shape[0])


def _blocks_for(length: int, block_size: int) -> int:
    return -(-int(length) // block_size)


def _place(pool: np.ndarray, table_row: np.ndarray, tokens_bits: np.ndarray, block_size: int) -> None:
    """Store tokens ``[n, Hkv, D]`` (positions 0..n-1) into the listed blocks.

    Positions fill blocks in order, ``block_size`` tokens per block; the tail of
    the last block keeps whatever the pool held.
    """
    n = tokens_bits.shape[0]
    if n == 0:
        return
    nb = _blocks_for(n, block_size)
    full = (n // block_size) * block_size
    if full:
        tiles = tokens_bits[:full].reshape(full // block_size, block_size, *tokens_bits.shape[1:])
        pool[table_row[: full // block_size]] = tiles.transpose(0, 2, 1, 3)
    if full < n:
        pool[table_row[nb - 1], :, : n - full, :] = tokens_bits[full:].transpose(1, 0, 2)


def _slot(table_row: np.ndarray, position: int, block_size: int) -> int:
    return int(table_row[position // block_size]) * block_size + position % block_size


def build_batch(
    name: str,
    *,
    seed: int,
    rng: np.random.Generator,
    dtype: str,
    num_q_heads: int,
    num_kv_heads: int,
    head_dim: int,
    block_size: int,
    context_lens,
    scale: float | None = None,
    pool_slack: float = 0.10,
    num_blocks: int | None = None,
    key_outlier_frac: float = 0.0,
    key_outlier_scale: float = 8.0,
    write_new_token: bool = True,
    partition_size: int = 0,
) -> PagedBatch:
    """Build a batch whose sequences own disjoint blocks of a shuffled pool.

    ``write_new_token``: the token at position ``L-1`` of every non-empty
    sequence is left out of the pool (its slot keeps the poison value) and is
    returned in ``key``/``value``/``slot_mapping`` instead, so a decode step
    first writes it and then attends over all ``L`` tokens.
    """
    assert dtype in DTYPES
    lens = np.asarray(context_lens, dtype=np.int64)
    S = lens.shape[0]
    B = block_size
    nbs = np.array([_blocks_for(L, B) for L in lens], dtype=np.int64)
    used = int(nbs.sum())
    N = int(num_blocks) if num_blocks is not None else max(1, math.ceil((1.0 + pool_slack) * used))
    assert N >= used, "pool too small"
    perm = rng.permutation(N).astype(np.int32)

    max_blocks = max(1, int(nbs.max()) if S else 1)
    tables = np.full((S, max_blocks), -1, dtype=np.int32)
    off = 0
    for s in range(S):
        tables[s, : nbs[s]] = perm[off : off + nbs[s]]
        off += int(nbs[s])

    poison = POISON_BITS[dtype]
    k_cache = np.full((N, num_kv_heads, B, head_dim), poison, dtype=np.uint16)
    v_cache = np.full_like(k_cache, poison)
    new_k, new_v, slots = [], [], []
    for s in range(S):
        L = int(lens[s])
        if L == 0:
            continue
        k = rng.standard_normal((L, num_kv_heads, head_dim), dtype=np.float32)
        v = rng.standard_normal((L, num_kv_heads, head_dim), dtype=np.float32)
        if key_outlier_frac > 0.0:
            picked = rng.random((L, num_kv_heads)) < key_outlier_frac
            k[picked] *= np.float32(key_outlier_scale)
        kb, vb = to_bits(k, dtype), to_bits(v, dtype)
        stored = L - 1 if write_new_token else L
        _place(k_cache, tables[s], kb[:stored], B)
        _place(v_cache, tables[s], vb[:stored], B)
        if write_new_token:
            new_k.append(kb[L - 1])
            new_v.append(vb[L - 1])
            slots.append(_slot(tables[s], L - 1, B))
    q = to_bits(rng.standard_normal((S, num_q_heads, head_dim), dtype=np.float32), dtype)

    shape_new = (0, num_kv_heads, head_dim)
    key = np.stack(new_k) if new_k else np.zeros(shape_new, np.uint16)
    value = np.stack(new_v) if new_v else np.zeros(shape_new, np.uint16)
    return PagedBatch(
        name=name,
        dtype=dtype,
        num_q_heads=num_q_heads,
        num_kv_heads=num_kv_heads,
        head_dim=head_dim,
        block_size=B,
        scale=float(scale if scale is not None else 1.0 / math.sqrt(head_dim)),
        q=q,
        k_cache=k_cache,
        v_cache=v_cache,
        block_tables=tables,
        context_lens=lens.astype(np.int32),
        key=key,
        value=value,
        slot_mapping=np.asarray(slots, dtype=np.int64),
        partition_size=partition_size,
        seed=seed,
    )


# --------------------------------------------------------------------------
# The five named workloads.
# --------------------------------------------------------------------------


def tiny(seed: int = 1) -> PagedBatch:
    """4 sequences, 4 q = 4 kv heads, head_dim 64, 16-token blocks, fp16,
    context lengths {1, 15, 16, 33}, a 16-block pool dealt in a seeded random
    order, scale 1/8, one new token per sequence written before attention."""
    rng = np.random.default_rng(seed)
    return build_batch(
        "tiny", seed=seed, rng=rng, dtype=F16, num_q_heads=4, num_kv_heads=4, head_dim=64,
        block_size=16, context_lens=[1, 15, 16, 33], num_blocks=16, scale=1.0 / 8.0,
    )


def llama7b_mha(seed: int = 2) -> PagedBatch:
    """Llama-7B-shaped multi-head decode layer: 64 sequences, 32 = 32 heads,
    head_dim 128, 16-token blocks, fp16, context lengths uniform on
    [128, 2048], pool = needed blocks + 10 %, shuffled."""
    rng = np.random.default_rng(seed)
    lens = rng.integers(128, 2048, size=64, endpoint=True)
    return build_batch(
        "llama7b_mha", seed=seed, rng=rng, dtype=F16, num_q_heads=32, num_kv_heads=32,
        head_dim=128, block_size=16, context_lens=lens,
    )


def lognormal_lengths(rng: np.random.Generator, n: int, mean: float, sigma: float, lo: int, hi: int) -> np.ndarray:
    """Lengths whose (unclipped) arithmetic mean is ``mean``: mu = ln(mean) - sigma^2/2."""
    mu = math.log(mean) - 0.5 * sigma * sigma
    return np.clip(np.rint(rng.lognormal(mu, sigma, size=n)), lo, hi).astype(np.int64)


def gqa_write(seed: int = 3) -> PagedBatch:
    """Grouped-query decode with cache write: 256 sequences, 32 q / 8 kv heads,
    head_dim 128, bf16, 16-token blocks, lengths lognormal (mean 512,
    sigma 0.8) clipped to [16, 4096]; 256 new tokens written before attention."""
    rng = np.random.default_rng(seed)
    lens = lognormal_lengths(rng, 256, 512.0, 0.8, 16, 4096)
    return build_batch(
        "gqa_write", seed=seed, rng=rng, dtype=BF16, num_q_heads=32, num_kv_heads=8,
        head_dim=128, block_size=16, context_lens=lens,
    )


def long_context(seed: int = 5) -> PagedBatch:
    """Long-context decode: 4 sequences of 131072 tokens, 32 q / 8 kv heads,
    head_dim 128, bf16, 32-token blocks, 1 % of key vectors scaled by 8,
    split into 512-token partitions."""
    rng = np.random.default_rng(seed)
    return build_batch(
        "long_context", seed=seed, rng=rng, dtype=BF16, num_q_heads=32, num_kv_heads=8,
        head_dim=128, block_size=32, context_lens=[131072] * 4, key_outlier_frac=0.01,
        key_outlier_scale=8.0, partition_size=512,
    )


def prefix_share(seed: int = 4, *, num_seqs: int = 128, prefix_tokens: int = 1024,
                 suffix_range=(64, 512), num_q_heads: int = 32, num_kv_heads: int = 8,
                 head_dim: int = 128, block_size: int = 16, dtype: str = F16) -> PagedBatch:
    """Sequences sharing one prompt prefix through the same physical blocks.

    Every sequence's table starts with the same ``ceil(prefix/B)`` shared
    blocks; its private suffix (uniform on ``suffix_range`` tokens) lives in
    blocks of its own.  The last shared block is the one each sequence copies
    on write: ``cow_pairs[s] = (shared last block, fresh block of seq s)``, and
    ``block_tables`` already points at the fresh copies
    (``block_tables_before_cow`` still points at the shared block).

    With a prefix that ends mid-block, the suffix tokens that fall into the
    copied block are not in the pool: they are this step's new tokens
    (``key``/``value``/``slot_mapping``, slots in each sequence's own copy),
    together with the last token of every sequence.  With a block-aligned
    prefix only the last token of every sequence is new.
    """
    rng = np.random.default_rng(seed)
    B = block_size
    S = num_seqs
    suffix = rng.integers(suffix_range[0], suffix_range[1], size=S, endpoint=True)
    lens = prefix_tokens + suffix
    n_shared = _blocks_for(prefix_tokens, B)
    partial = prefix_tokens % B  # tokens of the prefix in the last shared block
    fill_in_copy = (B - partial) % B  # suffix tokens that land in the copied block
    nbs = np.array([_blocks_for(L, B) for L in lens])
    private_after_shared = nbs - n_shared  # suffix blocks beyond the shared range
    used = n_shared + int(private_after_shared.sum()) + S  # + one CoW copy per seq
    N = math.ceil(1.10 * used)
    perm = rng.permutation(N).astype(np.int32)
    shared = perm[:n_shared]
    copies = perm[n_shared : n_shared + S]
    off = n_shared + S
    max_blocks = int(nbs.max())
    before = np.full((S, max_blocks), -1, dtype=np.int32)
    after = np.full_like(before, -1)
    for s in range(S):
        row = np.concatenate([shared, perm[off : off + private_after_shared[s]]])
        off += int(private_after_shared[s])
        before[s, : nbs[s]] = row
        row = row.copy()
        row[n_shared - 1] = copies[s]
        after[s, : nbs[s]] = row

    poison = POISON_BITS[dtype]
    k_cache = np.full((N, num_kv_heads, B, head_dim), poison, dtype=np.uint16)
    v_cache = np.full_like(k_cache, poison)
    kp = to_bits(rng.standard_normal((prefix_tokens, num_kv_heads, head_dim), dtype=np.float32), dtype)
    vp = to_bits(rng.standard_normal((prefix_tokens, num_kv_heads, head_dim), dtype=np.float32), dtype)
    _place(k_cache, shared, kp, B)
    _place(v_cache, shared, vp, B)
    new_k, new_v, slots = [], [], []
    for s in range(S):
        n_suf = int(suffix[s])
        ks = to_bits(rng.standard_normal((n_suf, num_kv_heads, head_dim), dtype=np.float32), dtype)
        vs = to_bits(rng.standard_normal((n_suf, num_kv_heads, head_dim), dtype=np.float32), dtype)
        # Suffix positions prefix+i; those in the copied block and the last
        # one are new this step, the rest sit in the private blocks already.
        new_idx = list(range(min(fill_in_copy, n_suf)))
        if (n_suf - 1) not in new_idx:
            new_idx.append(n_suf - 1)
        for i in new_idx:
            new_k.append(ks[i])
            new_v.append(vs[i])
            slots.append(_slot(after[s], prefix_tokens + i, B))
        # Stored suffix tokens beyond the copied block: positions from the
        # first private block boundary up to L-2.
        first_private_pos = n_shared * B
        stored_hi = prefix_tokens + n_suf - 1  # exclusive: last token is new
        if stored_hi > first_private_pos:
            lo = first_private_pos - prefix_tokens
            hi = stored_hi - prefix_tokens
            priv_row = after[s, n_shared : nbs[s]]
            _place(k_cache, priv_row, ks[lo:hi], B)
            _place(v_cache, priv_row, vs[lo:hi], B)
    q = to_bits(rng.standard_normal((S, num_q_heads, head_dim), dtype=np.float32), dtype)
    pairs = np.stack([np.full(S, shared[-1], np.int64), copies.astype(np.int64)], axis=1)
    return PagedBatch(
        name="prefix_share", dtype=dtype, num_q_heads=num_q_heads, num_kv_heads=num_kv_heads,
        head_dim=head_dim, block_size=B, scale=1.0 / math.sqrt(head_dim), q=q,
        k_cache=k_cache, v_cache=v_cache, block_tables=after, context_lens=lens.astype(np.int32),
        key=np.stack(new_k), value=np.stack(new_v), slot_mapping=np.asarray(slots, np.int64),
        cow_pairs=pairs, block_tables_before_cow=before, seed=seed,
    )


def small_case(seed: int, *, num_seqs: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
               block_size: int, dtype: str, max_len: int, min_len: int = 1,
               partition_size: int = 0, key_outlier_frac: float = 0.0,
               write_new_token: bool = True, lens=None) -> PagedBatch:
    """Reduced-size batch for parity tests: ragged lengths uniform on
    [min_len, max_len] unless ``lens`` is given."""
    rng = np.random.default_rng(seed)
    if lens is None:
        lens = rng.integers(min_len, max_len, size=num_seqs, endpoint=True)
    return build_batch(
        f"small_{seed}", seed=seed, rng=rng, dtype=dtype, num_q_heads=num_q_heads,
        num_kv_heads=num_kv_heads, head_dim=head_dim, block_size=block_size,
        context_lens=lens, key_outlier_frac=key_outlier_frac,
        write_new_token=write_new_token, partition_size=partition_size,
    )


WORKLOADS = {
    "tiny": tiny,
    "llama7b_mha": llama7b_mha,
    "gqa_write": gqa_write,
    "prefix_share": prefix_share,
    "long_context": long_context,
}


def shard_batch(batch: PagedBatch, rank: int, world: int) -> PagedBatch:
    """The sequences of one data-parallel shard, with a pool of their own.

    Sequences are split into ``world`` contiguous ranges; shard ``rank`` keeps
    its range, only the blocks those sequences reference (renumbered in
    order of first use), and their new tokens and copy pairs.  Pure data
    movement: the shard's decode outputs are the global batch's rows.
    """
    S = batch.num_seqs
    lo, hi = (S * rank) // world, (S * (rank + 1)) // world
    tables = batch.block_tables[lo:hi]
    before = None if batch.block_tables_before_cow is None else batch.block_tables_before_cow[lo:hi]
    used = [b for b in tables.ravel().tolist() if b >= 0]
    if before is not None:
        used += [b for b in before.ravel().tolist() if b >= 0]
    keep = list(dict.fromkeys(used))  # first-use order, unique
    remap = {b: i for i, b in enumerate(keep)}

    def rt(t):
        return np.vectorize(lambda b: remap.get(int(b), -1), otypes=[np.int32])(t) if t.size else t

    N = max(1, len(keep))
    kc = batch.k_cache[keep] if keep else batch.k_cache[:1]
    vc = batch.v_cache[keep] if keep else batch.v_cache[:1]
    B = batch.block_size
    slot_block = batch.slot_mapping // B
    tok = np.array([b in remap for b in slot_block.tolist()], dtype=bool)
    slots = np.array([remap[int(b)] * B + int(s) % B for b, s in zip(slot_block[tok], batch.slot_mapping[tok])],
                     dtype=np.int64)
    pairs = [(remap[int(a)], remap[int(b)]) for a, b in batch.cow_pairs.tolist()
             if int(a) in remap and int(b) in remap]
    return PagedBatch(
        name=f"{batch.name}[{rank}/{world}]", dtype=batch.dtype, num_q_heads=batch.num_q_heads,
        num_kv_heads=batch.num_kv_heads, head_dim=batch.head_dim, block_size=B, scale=batch.scale,
        q=batch.q[lo:hi], k_cache=np.ascontiguousarray(kc), v_cache=np.ascontiguousarray(vc),
        block_tables=rt(tables), context_lens=batch.context_lens[lo:hi],
        key=batch.key[tok], value=batch.value[tok], slot_mapping=slots,
        cow_pairs=np.asarray(pairs, dtype=np.int64).reshape(-1, 2),
        block_tables_before_cow=None if before is None else rt(before),
        partition_size=batch.partition_size, seed=batch.seed,
    )


# --------------------------------------------------------------------------
# 8-bit (E4M3) pools
# --------------------------------------------------------------------------
FP8_POISON = 0x7F  # an E4M3 NaN code


def random_e4m3_codes(rng: np.random.Generator, shape, exp_lo: int = 4, exp_hi: int = 10) -> np.ndarray:
    """Random E4M3 codes drawn field by field (no rounding involved): a random
    sign, an exponent field uniform on [exp_lo, exp_hi] and a uniform 3-bit
    mantissa; magnitudes span 2^(exp_lo-7) .. 1.875 * 2^(exp_hi-7)."""
    sign = rng.integers(0, 2, size=shape, dtype=np.uint8) << 7
    exp = rng.integers(exp_lo, exp_hi + 1, size=shape, dtype=np.uint8) << 3
    man = rng.integers(0, 8, size=shape, dtype=np.uint8)
    return (sign | exp | man).astype(np.uint8)


@dataclass
class Fp8Batch:
    """A decode step over 8-bit pools: the fp16/bf16 batch's queries, new
    tokens, tables and lengths, with K [N][Hkv][B][D] and V [N][Hkv][D][B]
    pools of E4M3 codes and one scale per pool."""

    base: PagedBatch
    k_cache: np.ndarray  # uint8 [N, Hkv, B, D]
    v_cache: np.ndarray  # uint8 [N, Hkv, D, B]
    k_scale: float
    v_scale: float

    def __getattr__(self, name):
        return getattr(self.base, name)


def all_finite_e4m3_codes(rng: np.random.Generator, shape) -> np.ndarray:
    """Random E4M3 codes uniform over all 254 finite codes (every exponent
    field 0..15, subnormals and both zeros included; only the two NaN codes
    0x7F and 0xFF are left out)."""
    c = rng.integers(0, 254, size=shape, dtype=np.int32)
    return (c + (c >= 0x7F)).astype(np.uint8)


def fp8_variant(batch: PagedBatch, seed: int, k_scale: float = 0.125, v_scale: float = 0.0625,
                full_range: bool = False) -> Fp8Batch:
    """Replace the pools of ``batch`` by 8-bit pools: every position a sequence
    attends to (except this step's new tokens, which the step writes) holds a
    random code; every other slot holds the NaN code.  Codes have exponent
    fields 4..10 (``random_e4m3_codes``), or with ``full_range`` are uniform
    over all 254 finite codes."""
    rng = np.random.default_rng(seed)
    draw = all_finite_e4m3_codes if full_range else random_e4m3_codes
    N, Hkv, B, D = batch.k_cache.shape
    kc = np.full((N, Hkv, B, D), FP8_POISON, dtype=np.uint8)
    vc = np.full((N, Hkv, D, B), FP8_POISON, dtype=np.uint8)
    for s in range(batch.num_seqs):
        L = int(batch.context_lens[s])
        if L == 0:
            continue
        kt = draw(rng, (L, Hkv, D))
        vt = draw(rng, (L, Hkv, D))
        nb = _blocks_for(L, B)
        pad = nb * B - L
        kp = np.concatenate([kt, np.full((pad, Hkv, D), FP8_POISON, np.uint8)]).reshape(nb, B, Hkv, D)
        vp = np.concatenate([vt, np.full((pad, Hkv, D), FP8_POISON, np.uint8)]).reshape(nb, B, Hkv, D)
        rows = batch.block_tables[s, :nb]
        kc[rows] = kp.transpose(0, 2, 1, 3)
        vc[rows] = vp.transpose(0, 2, 3, 1)
    for slot in batch.slot_mapping.tolist():  # slots this step writes start poisoned
        if slot >= 0:
            kc[slot // B, :, slot % B, :] = FP8_POISON
            vc[slot // B, :, :, slot % B] = FP8_POISON
    return Fp8Batch(base=batch, k_cache=kc, v_cache=vc, k_scale=k_scale, v_scale=v_scale)


# --------------------------------------------------------------------------
# Chunked-prefill batches
# --------------------------------------------------------------------------


@dataclass
class PrefillBatch:
    """One prefill call: sequence s has ``context_lens[s]`` tokens, the last
    ``chunk_lens[s]`` of which are this call's new tokens (queries ``q`` rows
    ``query_start[s] .. query_start[s+1]``; their K/V in ``key``/``value``,
    to be written to ``slot_mapping`` before attention).  Earlier tokens are
    already in the pools; every other slot holds the poison value."""

    name: str
    dtype: str
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    scale: float
    q: np.ndarray            # [T, Hq, D] bits
    k_cache: np.ndarray      # [N, Hkv, B, D] bits
    v_cache: np.ndarray
    block_tables: np.ndarray  # [S, max_blocks] int32, -1 padded
    context_lens: np.ndarray  # [S] int32
    query_start: np.ndarray   # [S + 1] int32
    key: np.ndarray           # [T, Hkv, D] bits
    value: np.ndarray
    slot_mapping: np.ndarray  # [T] int64
    seed: int

    @property
    def num_seqs(self) -> int:
        return int(self.context_lens.shape[0])

    @property
    def num_tokens(self) -> int:
        return int(self.q.shape[0])

    @property
    def chunk_lens(self) -> np.ndarray:
        return np.diff(self.query_start)

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max()) if self.num_seqs else 0

    @property
    def max_query_len(self) -> int:
        return int(self.chunk_lens.max()) if self.num_seqs else 0


def prefill_batch(seed: int, *, dtype: str, num_q_heads: int, num_kv_heads: int, head_dim: int,
                  block_size: int, context_lens, chunk_lens, scale: float | None = None,
                  pool_slack: float = 0.10, name: str | None = None) -> PrefillBatch:
    """Sequences own disjoint blocks of a shuffled pool; q, K, V ~ N(0, 1)."""
    assert dtype in DTYPES
    rng = np.random.default_rng(seed)
    lens = np.asarray(context_lens, dtype=np.int64)
    chunks = np.asarray(chunk_lens, dtype=np.int64)
    assert lens.shape == chunks.shape and np.all(chunks <= lens) and np.all(chunks >= 0)
    S, B = lens.shape[0], block_size
    nbs = np.array([_blocks_for(L, B) for L in lens], dtype=np.int64)
    used = int(nbs.sum())
    N = max(1, math.ceil((1.0 + pool_slack) * used))
    perm = rng.permutation(N).astype(np.int32)
    tables = np.full((S, max(1, int(nbs.max()) if S else 1)), -1, dtype=np.int32)
    off = 0
    for s in range(S):
        tables[s, : nbs[s]] = perm[off : off + nbs[s]]
        off += int(nbs[s])
    poison = POISON_BITS[dtype]
    k_cache = np.full((N, num_kv_heads, B, head_dim), poison, dtype=np.uint16)
    v_cache = np.full_like(k_cache, poison)
    new_k, new_v, slots = [], [], []
    for s in range(S):
        L, C = int(lens[s]), int(chunks[s])
        kb = to_bits(rng.standard_normal((L, num_kv_heads, head_dim), dtype=np.float32), dtype)
        vb = to_bits(rng.standard_normal((L, num_kv_heads, head_dim), dtype=np.float32), dtype)
        _place(k_cache, tables[s], kb[: L - C], B)
        _place(v_cache, tables[s], vb[: L - C], B)
        new_k.append(kb[L - C:])
        new_v.append(vb[L - C:])
        slots += [_slot(tables[s], p, B) for p in range(L - C, L)]
    T = int(chunks.sum())
    q = to_bits(rng.standard_normal((T, num_q_heads, head_dim), dtype=np.float32), dtype)
    shape0 = (0, num_kv_heads, head_dim)
    return PrefillBatch(
        name=name or f"prefill_{seed}", dtype=dtype, num_q_heads=num_q_heads, num_kv_heads=num_kv_heads,
        head_dim=head_dim, block_size=B, scale=float(scale if scale is not None else 1.0 / math.sqrt(head_dim)),
        q=q, k_cache=k_cache, v_cache=v_cache, block_tables=tables, context_lens=lens.astype(np.int32),
        query_start=np.concatenate([[0], np.cumsum(chunks)]).astype(np.int32),
        key=np.concatenate(new_k) if T else np.zeros(shape0, np.uint16),
        value=np.concatenate(new_v) if T else np.zeros(shape0, np.uint16),
        slot_mapping=np.asarray(slots, dtype=np.int64), seed=seed,
    )


def prefill_llama7b(seed: int = 6) -> PrefillBatch:
    """Llama-7B-shaped multi-head prefill: 4 prompts of 4096 tokens, 32 = 32
    heads, head_dim 128, 16-token blocks, fp16; the whole prompt is the chunk."""
    return prefill_batch(seed, dtype=F16, num_q_heads=32, num_kv_heads=32, head_dim=128, block_size=16,
                         context_lens=[4096] * 4, chunk_lens=[4096] * 4, name="prefill_llama7b")


def prefill_gqa_chunked(seed: int = 7) -> PrefillBatch:
    """Chunked prefill with grouped-query heads: 8 sequences whose 1024-token
    chunks end 8192-token contexts (7168 tokens already cached), 32 q / 8 kv
    heads, head_dim 128, 16-token blocks, bf16."""
    return prefill_batch(seed, dtype=BF16, num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=16,
                         context_lens=[8192] * 8, chunk_lens=[1024] * 8, name="prefill_gqa_chunked")


def prefill_mixed(seed: int = 11) -> PrefillBatch:
    """A mixed serving batch: 16 sequences whose chunks are 64..2048 tokens
    (uniform) on top of 0..6000 cached tokens (uniform), 32 q / 8 kv heads,
    head_dim 128, 16-token blocks, bf16.  The work per (sequence, kv head)
    differs by up to ~100x, which is what an even spread of work over the
    SMs has to absorb."""
    r = np.random.default_rng(seed)
    C = r.integers(64, 2049, 16)
    L = C + r.integers(0, 6001, 16)
    return prefill_batch(seed, dtype=BF16, num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=16,
                         context_lens=[int(x) for x in L], chunk_lens=[int(x) for x in C], name="prefill_mixed")


PREFILL_WORKLOADS = {
    "prefill_llama7b": prefill_llama7b,
    "prefill_gqa_chunked": prefill_gqa_chunked,
    "prefill_mixed": prefill_mixed,
}
