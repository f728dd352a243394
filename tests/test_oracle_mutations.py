"""Plant plausible mistakes in the oracle (on the CPU) and confirm that at
least one pin catches each of them."""

import numpy as np
import pytest

import oracle.block_manager as BMO
import oracle.paged_kv as O
import oracle.prefill as PO
from pins import ALL_CHECKS

_orig_attend = O.attend
_orig_materialize = O.materialize
_orig_lse = O.lse_combine


def _attend_no_scale(q, K, V, scale):
    return _orig_attend(q, K, V, 1.0)


def _attend_values_from_keys(q, K, V, scale):
    return _orig_attend(q, K, K, scale)


def _attend_softmax_wrong_axis(q, K, V, scale):
    q = np.asarray(q, dtype=np.float64)
    if K.shape[0] == 0:
        return np.zeros((q.shape[0], V.shape[1]))
    z = scale * (q @ K.T)
    e = np.exp(z - z.max(axis=0, keepdims=True))
    return (e / e.sum(axis=0, keepdims=True)) @ V


def _attend_drop_last_token(q, K, V, scale):
    return _orig_attend(q, K[:-1] if K.shape[0] > 1 else K, V[:-1] if V.shape[0] > 1 else V, scale)


def _materialize_offset_shift(cache, table_row, length, block_size):
    pos = np.arange(length)
    blocks = np.asarray(table_row)[pos // block_size].astype(np.int64)
    offs = (pos + 1) % block_size
    return np.ascontiguousarray(cache[blocks, :, offs, :].transpose(1, 0, 2))


def _materialize_heads_swapped(cache, table_row, length, block_size):
    return _orig_materialize(cache, table_row, length, block_size)[::-1].copy()


def _kv_head_modulo(h, num_q_heads, num_kv_heads):
    return h % num_kv_heads


def _slot_location_swapped(slot, block_size):
    return int(slot) % block_size, int(slot) // block_size


def _copy_blocks_reversed(k_cache, v_cache, block_pairs):
    pairs = np.asarray(block_pairs).reshape(-1, 2)[:, ::-1]
    k0, v0 = np.array(k_cache), np.array(v_cache)
    kc, vc = k0.copy(), v0.copy()
    for src, dst in pairs.tolist():
        kc[dst], vc[dst] = k0[src], v0[src]
    return kc, vc


def _lse_unweighted_l(ms, ls, os):
    M = ms.max(axis=0)
    w = np.exp(ms - M)
    w = np.where(np.isfinite(w), w, 0.0)
    return (w[:, :, None] * os).sum(axis=0) / ls.sum(axis=0)[:, None]


def _append_always_new_block(table, length, free_pool, block_size):
    table.append(free_pool.pop(0))
    return table[-1] * block_size


def _encode_truncate(x, dtype):
    x = np.asarray(x, dtype=np.float64)
    if dtype == O.BF16:
        return (x.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    return x.astype(np.float16).view(np.uint16)


_orig_e4m3 = O.e4m3_encode


def _e4m3_truncating(x):
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, ex = np.frexp(a)
    q = np.ldexp(np.floor(np.ldexp(a, -(np.maximum(ex - 1, -6) - 3))), np.maximum(ex - 1, -6) - 3)
    return _orig_e4m3(np.copysign(q, x))


def _materialize_fp8_v_untransposed(k_cache, v_cache, table_row, length, block_size):
    pos = np.arange(length)
    blocks = np.asarray(table_row)[pos // block_size].astype(np.int64)
    offs = pos % block_size
    K = k_cache[blocks, :, offs, :]
    V = v_cache[blocks, :, offs, :]  # reads a dimension row as if it were a token row
    return np.ascontiguousarray(K.transpose(1, 0, 2)), np.ascontiguousarray(V.transpose(1, 0, 2))


def _bm_append_in_place(self, seq_ids):
    """Copy-on-write left out: a shared last block is written in place."""
    seq_ids = list(seq_ids)
    B = self.block_size
    slots = []
    for s in seq_ids:
        table, L = self.tables[s], self.lens[s]
        if L % B == 0:
            table.append(self._take())
        slots.append(table[-1] * B + L % B)
        self.lens[s] = L + 1
    return slots, []


def _bm_free_ignores_refs(self, seq_id):
    for b in self.tables.pop(seq_id):
        self.ref[b] = 0
        if b not in self.free:
            self.free.append(b)
    del self.lens[seq_id]


def _bm_fork_without_refs(self, parent, child):
    self.tables[child] = list(self.tables[parent])
    self.lens[child] = self.lens[parent]


def _bm_needed_counts_every_shared(self, seq_ids):
    B = self.block_size
    return sum(1 for s in seq_ids if self.lens[s] % B == 0 or self.ref[self.tables[s][-1]] > 1)


def _prefill_not_causal(q_bits, k_cache, v_cache, block_tables, query_start, context_lens, block_size, scale,
                        dtype, seqs=None):
    """Every chunk token attends over the whole sequence."""
    T, Hq, D = q_bits.shape
    Hkv = k_cache.shape[1]
    out = np.full((T, Hq, D), np.nan)
    for s in range(len(context_lens)):
        t0, t1, L = int(query_start[s]), int(query_start[s + 1]), int(context_lens[s])
        K = O.decode_bits(O.materialize(k_cache, block_tables[s], L, block_size), dtype)
        V = O.decode_bits(O.materialize(v_cache, block_tables[s], L, block_size), dtype)
        for t in range(t0, t1):
            q = O.decode_bits(q_bits[t], dtype)
            for h in range(Hq):
                g = O.kv_head_of(h, Hq, Hkv)
                out[t, h] = O.attend(q[h:h + 1], K[g], V[g], scale)[0]
    return out


def _prefill_excludes_itself(q_bits, k_cache, v_cache, block_tables, query_start, context_lens, block_size,
                             scale, dtype, seqs=None):
    """Each token sees only the positions before it (the first sees itself)."""
    T, Hq, D = q_bits.shape
    Hkv = k_cache.shape[1]
    out = np.full((T, Hq, D), np.nan)
    for s in range(len(context_lens)):
        t0, t1, L = int(query_start[s]), int(query_start[s + 1]), int(context_lens[s])
        K = O.decode_bits(O.materialize(k_cache, block_tables[s], L, block_size), dtype)
        V = O.decode_bits(O.materialize(v_cache, block_tables[s], L, block_size), dtype)
        for j, t in enumerate(range(t0, t1)):
            p = max(1, L - (t1 - t0) + j)
            q = O.decode_bits(q_bits[t], dtype)
            for h in range(Hq):
                g = O.kv_head_of(h, Hq, Hkv)
                out[t, h] = O.attend(q[h:h + 1], K[g, :p], V[g, :p], scale)[0]
    return out


PREFILL_MUTANTS = {
    "prefill_not_causal": ("paged_prefill", _prefill_not_causal),
    "prefill_query_excludes_itself": ("paged_prefill", _prefill_excludes_itself),
}

BM_MUTANTS = {
    "manager_copy_on_write_left_out": ("append", _bm_append_in_place),
    "manager_free_ignores_refcounts": ("free_sequence", _bm_free_ignores_refs),
    "manager_fork_takes_no_reference": ("fork", _bm_fork_without_refs),
    "manager_step_count_ignores_earlier_copies": ("blocks_needed", _bm_needed_counts_every_shared),
}

MUTANTS = {
    "attend_drops_scale": ("attend", _attend_no_scale),
    "attend_uses_keys_as_values": ("attend", _attend_values_from_keys),
    "softmax_over_wrong_axis": ("attend", _attend_softmax_wrong_axis),
    "attend_drops_last_token": ("attend", _attend_drop_last_token),
    "gather_offset_off_by_one": ("materialize", _materialize_offset_shift),
    "gather_heads_reversed": ("materialize", _materialize_heads_swapped),
    "gqa_modulo_grouping": ("kv_head_of", _kv_head_modulo),
    "slot_block_offset_swapped": ("slot_location", _slot_location_swapped),
    "copy_blocks_direction_reversed": ("copy_blocks", _copy_blocks_reversed),
    "lse_combine_unweighted_sum": ("lse_combine", _lse_unweighted_l),
    "append_without_filling_block": ("append_token", _append_always_new_block),
    "bf16_truncates_instead_of_rounding": ("encode_bits", _encode_truncate),
    "e4m3_truncates_instead_of_rounding": ("e4m3_encode", _e4m3_truncating),
    "fp8_v_pool_read_untransposed": ("materialize_fp8", _materialize_fp8_v_untransposed),
}


@pytest.mark.parametrize("name", sorted(MUTANTS) + sorted(BM_MUTANTS) + sorted(PREFILL_MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    if name in BM_MUTANTS:
        attr, fn = BM_MUTANTS[name]
        monkeypatch.setattr(BMO.BlockManager, attr, fn)
    elif name in PREFILL_MUTANTS:
        attr, fn = PREFILL_MUTANTS[name]
        monkeypatch.setattr(PO, attr, fn)
    else:
        attr, fn = MUTANTS[name]
        monkeypatch.setattr(O, attr, fn)
    caught = []
    for check in ALL_CHECKS:
        try:
            check()
        except AssertionError:
            caught.append(check.__name__)
        except (IndexError, ValueError, KeyError, BMO.OutOfBlocks):
            caught.append(check.__name__ + " (raised)")
    assert caught, f"no pin catches the planted mistake {name}"
