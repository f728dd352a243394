"""Pins of the oracle to facts outside itself.

Each ``check_*`` raises AssertionError when the oracle disagrees with what the
pages, the mathematics or an independent computation fix.  They call the oracle
through the module attribute (``O.name``) at call time, so a test can plant a
mistake in the oracle with ``monkeypatch`` and confirm some check catches it.
"""

from __future__ import annotations

import math
import os

import numpy as np

import oracle.paged_kv as O
import workloads as W
from conftest import read_fixture

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rand_bits(rng, shape, dtype):
    return W.to_bits(rng.standard_normal(shape, dtype=np.float32), dtype)


# ---------------------------------------------------------------------------
# Paging: block table, append rule, gather
# ---------------------------------------------------------------------------

def check_block_table_example():
    """The page's Block Tables A = [3, 7, 12] and B = [1, 5, 9, 14]: tag every
    (block, position) of a 16-block pool with a unique code and read the
    requests back through their tables.  The expected sequences are written
    block by block from the tables (16 tokens per block, in table order)."""
    fx = read_fixture(os.path.join(GOLDEN, "block_table_example.txt"))
    B = fx["block_size"][0]
    pool = np.zeros((16, 1, B, 1), dtype=np.uint16)
    for b in range(16):
        for o in range(B):
            pool[b, 0, o, 0] = b * 100 + o
    exp_a = [300 + o for o in range(16)] + [700 + o for o in range(16)] + [1200 + o for o in range(16)]
    exp_b = ([100 + o for o in range(16)] + [500 + o for o in range(16)]
             + [900 + o for o in range(16)] + [1400 + o for o in range(16)])
    for name, expected in (("table_A", exp_a), ("table_B", exp_b)):
        table = np.array(fx[name], dtype=np.int32)
        for length in (1, 15, 16, 17, 20, len(expected)):
            got = O.materialize(pool, table, length, B)[0, :, 0].tolist()
            assert got == expected[:length], (name, length)
    # token 20 of request A sits in its second block (Block7) at position 4
    assert O.materialize(pool, np.array(fx["table_A"]), 21, B)[0, 20, 0] == 704


def check_append_rule_example():
    fx = read_fixture(os.path.join(GOLDEN, "append_rule_example.txt"))
    B = fx["block_size"][0]
    free = list(fx["free_pool"])
    table, slots = [], []
    for t in range(fx["tokens"][0]):
        slots.append(O.append_token(table, t, free, B))
    assert table == fx["expect_table"]
    for t in (0, 15, 16, 31, 32):
        assert slots[t] == fx[f"expect_slot_token_{t}"][0], t
    assert free == [8]
    O.free_request(table, free)
    assert free == fx["expect_free_after_finish"] and table == []


def check_generator_follows_append_rule():
    """Replaying the append rule token by token, with each sequence's blocks
    as the free pool in table order, rebuilds the generated Block Tables and
    the slot of every sequence's new token."""
    batch = W.small_case(11, num_seqs=6, num_q_heads=4, num_kv_heads=2, head_dim=8,
                         block_size=8, dtype=W.F16, max_len=40)
    B = batch.block_size
    for s in range(batch.num_seqs):
        L = int(batch.context_lens[s])
        nb = -(-L // B)
        free = batch.block_tables[s, :nb].tolist()
        table, slot = [], None
        for t in range(L):
            slot = O.append_token(table, t, free, B)
        assert table == batch.block_tables[s, :nb].tolist()
        assert slot == int(batch.slot_mapping[s])


def check_materialize_roundtrip():
    """Scatter a contiguous sequence into a shuffled pool one block slice at a
    time; reading it back through the table returns it bit for bit."""
    rng = np.random.default_rng(7)
    for B, L in ((8, 1), (8, 8), (16, 37), (32, 100), (64, 64)):
        Hkv, D = 3, 16
        nb = -(-L // B)
        N = nb + 5
        table = rng.permutation(N)[:nb].astype(np.int32)
        seq = rng.integers(0, 2 ** 16, size=(Hkv, L, D)).astype(np.uint16)
        pool = rng.integers(0, 2 ** 16, size=(N, Hkv, B, D)).astype(np.uint16)
        start = 0
        for blk in table:
            stop = min(start + B, L)
            pool[blk, :, : stop - start, :] = seq[:, start:stop, :]
            start = stop
        assert np.array_equal(O.materialize(pool, table, L, B), seq), (B, L)


# ---------------------------------------------------------------------------
# Attention core: closed forms and special cases
# ---------------------------------------------------------------------------

def check_single_token_returns_value():
    rng = np.random.default_rng(1)
    q = rng.standard_normal((3, 16))
    K = rng.standard_normal((1, 16)) * 10
    V = rng.standard_normal((1, 16))
    out = O.attend(q, K, V, 0.37)
    assert np.array_equal(out, np.repeat(V, 3, axis=0))


def check_two_token_sigmoid():
    """With two keys the softmax weight of key 1 is the logistic function of
    the score difference: out = s(D) v1 + (1 - s(D)) v0, D = scale q.(k1 - k0)."""
    rng = np.random.default_rng(2)
    for _ in range(20):
        D = 8
        q = rng.standard_normal(D)
        K = rng.standard_normal((2, D)) * 2
        V = rng.standard_normal((2, D))
        scale = float(rng.uniform(0.05, 1.5))
        delta = scale * sum(q[i] * (K[1, i] - K[0, i]) for i in range(D))
        w1 = 1.0 / (1.0 + math.exp(-delta))
        expected = [w1 * V[1, i] + (1.0 - w1) * V[0, i] for i in range(D)]
        got = O.attend(q[None, :], K, V, scale)[0]
        assert np.allclose(got, expected, rtol=0, atol=1e-13)


def check_uniform_weights_give_mean():
    """Equal keys, or scale 0, make every weight 1/L: the output is the mean of V."""
    rng = np.random.default_rng(3)
    q = rng.standard_normal((2, 12))
    V = rng.standard_normal((9, 12))
    K_equal = np.repeat(rng.standard_normal((1, 12)), 9, axis=0)
    mean = V.sum(axis=0) / 9
    assert np.allclose(O.attend(q, K_equal, V, 0.8), mean[None, :], rtol=0, atol=1e-14)
    K = rng.standard_normal((9, 12))
    assert np.allclose(O.attend(q, K, V, 0.0), mean[None, :], rtol=0, atol=1e-14)


def check_dominant_key():
    """A key aligned with the query and far larger than the others takes all
    the weight: the output is that key's value (to within e^-gap)."""
    rng = np.random.default_rng(4)
    q = rng.standard_normal(16)
    K = rng.standard_normal((30, 16))
    K[17] = 40.0 * q / np.linalg.norm(q)
    V = rng.standard_normal((30, 16))
    out = O.attend(q[None, :], K, V, 1.0)[0]
    assert np.allclose(out, V[17], rtol=0, atol=1e-9)


def check_against_torch_sdpa():
    """Library special case: on the materialised sequences, decode attention
    equals torch's scaled_dot_product_attention in float64 on the CPU (grouped
    query heads expanded with ``repeat_interleave``)."""
    import torch

    for dtype in (W.F16, W.BF16):
        batch = W.small_case(21, num_seqs=5, num_q_heads=8, num_kv_heads=2, head_dim=32,
                             block_size=16, dtype=dtype, max_len=70, write_new_token=False)
        out = O.paged_attention_decode(batch.q, batch.k_cache, batch.v_cache, batch.block_tables,
                                       batch.context_lens, batch.block_size, batch.scale, dtype)
        G = batch.num_q_heads // batch.num_kv_heads
        for s in range(batch.num_seqs):
            L = int(batch.context_lens[s])
            K = O.decode_bits(O.materialize(batch.k_cache, batch.block_tables[s], L, 16), dtype)
            V = O.decode_bits(O.materialize(batch.v_cache, batch.block_tables[s], L, 16), dtype)
            q = torch.from_numpy(O.decode_bits(batch.q[s], dtype))[:, None, :]  # [Hq, 1, D]
            Kt = torch.from_numpy(K).repeat_interleave(G, dim=0)  # [Hq, L, D]
            Vt = torch.from_numpy(V).repeat_interleave(G, dim=0)
            ref = torch.nn.functional.scaled_dot_product_attention(q, Kt, Vt, scale=batch.scale)
            assert np.allclose(out[s], ref[:, 0, :].numpy(), rtol=0, atol=1e-12), (dtype, s)


def check_gqa_grouping():
    """Query head h reads kv head h // G: with V constant per kv head (value
    g+1), every output element of head h equals h // G + 1."""
    rng = np.random.default_rng(5)
    Hq, Hkv, D, B, L = 8, 2, 8, 8, 11
    N = 4
    table = np.array([2, 0], dtype=np.int32)
    k_cache = _rand_bits(rng, (N, Hkv, B, D), W.BF16)
    v_cache = np.zeros((N, Hkv, B, D), dtype=np.uint16)
    for g in range(Hkv):
        v_cache[:, g] = W.to_bits(np.full((N, B, D), g + 1, np.float32), W.BF16)
    q = _rand_bits(rng, (Hq, D), W.BF16)
    out = O.decode_sequence(q, k_cache, v_cache, table, L, B, 0.3, W.BF16)
    for h in range(Hq):
        assert np.allclose(out[h], h // (Hq // Hkv) + 1, rtol=0, atol=1e-14), h


def check_brute_force_tiny():
    """An independent pure-Python evaluation on a tiny batch: every key and
    value fetched token by token with its own table lookup, scores, softmax
    and weighted sum written as loops."""
    batch = W.small_case(31, num_seqs=3, num_q_heads=4, num_kv_heads=2, head_dim=4,
                         block_size=4, dtype=W.F16, max_len=11, write_new_token=False)
    out = O.paged_attention_decode(batch.q, batch.k_cache, batch.v_cache, batch.block_tables,
                                   batch.context_lens, batch.block_size, batch.scale, W.F16)
    Bs = batch.block_size
    f16 = lambda b: float(np.uint16(b).view(np.float16))  # noqa: E731
    for s in range(batch.num_seqs):
        L = int(batch.context_lens[s])
        for h in range(4):
            g = h // 2
            keys, vals = [], []
            for i in range(L):
                blk = int(batch.block_tables[s][i // Bs])
                keys.append([f16(batch.k_cache[blk, g, i % Bs, d]) for d in range(4)])
                vals.append([f16(batch.v_cache[blk, g, i % Bs, d]) for d in range(4)])
            qv = [f16(batch.q[s, h, d]) for d in range(4)]
            scores = [batch.scale * sum(qv[d] * k[d] for d in range(4)) for k in keys]
            top = max(scores)
            ws = [math.exp(z - top) for z in scores]
            tot = sum(ws)
            for d in range(4):
                ref = sum(ws[i] * vals[i][d] for i in range(L)) / tot
                assert abs(out[s, h, d] - ref) <= 1e-13, (s, h, d)


def check_empty_sequence_is_zero():
    rng = np.random.default_rng(6)
    out = O.attend(rng.standard_normal((2, 8)), np.zeros((0, 8)), np.zeros((0, 8)), 1.0)
    assert np.array_equal(out, np.zeros((2, 8)))


# ---------------------------------------------------------------------------
# Paging invariants
# ---------------------------------------------------------------------------

def _decode(batch, tables=None, k_cache=None, v_cache=None):
    return O.paged_attention_decode(
        batch.q, batch.k_cache if k_cache is None else k_cache,
        batch.v_cache if v_cache is None else v_cache,
        batch.block_tables if tables is None else tables, batch.context_lens,
        batch.block_size, batch.scale, batch.dtype)


def check_placement_invariance():
    """Physical storage is decoupled from the logical view: moving every block
    to another physical slot (and rewriting the tables) changes nothing."""
    batch = W.small_case(41, num_seqs=4, num_q_heads=4, num_kv_heads=4, head_dim=16,
                         block_size=8, dtype=W.BF16, max_len=60, write_new_token=False)
    base = _decode(batch)
    rng = np.random.default_rng(42)
    N = batch.num_blocks
    perm = rng.permutation(N)  # new home of block b is perm[b]
    k2 = np.empty_like(batch.k_cache)
    v2 = np.empty_like(batch.v_cache)
    k2[perm] = batch.k_cache
    v2[perm] = batch.v_cache
    t2 = np.where(batch.block_tables >= 0, perm[np.maximum(batch.block_tables, 0)], -1).astype(np.int32)
    assert np.array_equal(_decode(batch, t2, k2, v2), base)


def check_table_padding_ignored():
    """Table entries past a sequence's last block are never read: pointing them
    at other sequences' blocks changes nothing."""
    batch = W.small_case(43, num_seqs=5, num_q_heads=2, num_kv_heads=1, head_dim=8,
                         block_size=8, dtype=W.F16, max_len=50, write_new_token=False)
    base = _decode(batch)
    rng = np.random.default_rng(44)
    t2 = batch.block_tables.copy()
    pad = t2 < 0
    t2[pad] = rng.integers(0, batch.num_blocks, size=int(pad.sum()))
    assert np.array_equal(_decode(batch, t2), base)


def check_shared_prefix_equals_private_copy():
    """Sequences reading a shared prefix block give the same output as after
    copy-on-write gave each of them a private copy ([LSHU] 内存共享)."""
    batch = W.prefix_share(45, num_seqs=6, prefix_tokens=40, suffix_range=(3, 20), num_q_heads=4,
                           num_kv_heads=2, head_dim=16, block_size=16, dtype=W.F16)
    # Block-aligned?  40 % 16 = 8: the copied block also receives new tokens,
    # so compare on the pool state where no new token is written yet.
    kc, vc = O.copy_blocks(batch.k_cache, batch.v_cache, batch.cow_pairs)
    lens = batch.context_lens
    # Attend over the prefix plus the suffix tokens stored before this step,
    # i.e. up to the first position that is written in this step.
    first_new = np.array([40] * batch.num_seqs, dtype=np.int32)
    shared = O.paged_attention_decode(batch.q, kc, vc, batch.block_tables_before_cow, first_new,
                                      16, batch.scale, batch.dtype)
    private = O.paged_attention_decode(batch.q, kc, vc, batch.block_tables, first_new,
                                       16, batch.scale, batch.dtype)
    assert np.array_equal(shared, private)
    assert np.all(np.isfinite(shared))
    del lens


def check_split_lse_combine():
    """Merging the partial states of any partition of [0, L) reproduces the
    unsplit softmax attention."""
    rng = np.random.default_rng(8)
    for trial in range(30):
        L = int(rng.integers(1, 300))
        G, D = 4, 16
        q = rng.standard_normal((G, D))
        K = rng.standard_normal((L, D)) * (1 + 4 * (trial % 3 == 0))
        V = rng.standard_normal((L, D))
        cuts = sorted(set(rng.integers(0, L + 1, size=int(rng.integers(0, 6))).tolist()) | {0, L})
        parts = [O.partial_state(q, K[a:b], V[a:b], 0.2) for a, b in zip(cuts[:-1], cuts[1:])]
        parts.append(O.partial_state(q, K[:0], V[:0], 0.2))  # an empty partition
        ms = np.stack([p[0] for p in parts])
        ls = np.stack([p[1] for p in parts])
        os_ = np.stack([p[2] for p in parts])
        assert np.allclose(O.lse_combine(ms, ls, os_), O.attend(q, K, V, 0.2), rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------
# Cache write, block copy, storage formats
# ---------------------------------------------------------------------------

def check_reshape_and_cache_example():
    """Three new tokens with slots [5, -1, 18] in a pool of 8-token blocks:
    token 0 lands in block 0 position 5, token 1 is padding, token 2 lands in
    block 2 position 2; nothing else changes."""
    N, Hkv, B, D = 4, 2, 8, 4
    kc = np.full((N, Hkv, B, D), 0xAAAA, np.uint16)
    vc = np.full((N, Hkv, B, D), 0x5555, np.uint16)
    key = np.arange(3 * Hkv * D, dtype=np.uint16).reshape(3, Hkv, D) + 1
    value = key + 1000
    k2, v2 = O.reshape_and_cache(kc, vc, key, value, np.array([5, -1, 18]), B)
    ek, ev = kc.copy(), vc.copy()
    ek[0, :, 5, :] = key[0]
    ev[0, :, 5, :] = value[0]
    ek[2, :, 2, :] = key[2]
    ev[2, :, 2, :] = value[2]
    assert np.array_equal(k2, ek) and np.array_equal(v2, ev)
    assert np.all(kc == 0xAAAA)  # inputs untouched


def check_copy_blocks_example():
    N, Hkv, B, D = 6, 2, 4, 4
    kc = np.arange(N * Hkv * B * D, dtype=np.uint16).reshape(N, Hkv, B, D)
    vc = kc + 7
    k2, v2 = O.copy_blocks(kc, vc, np.array([[1, 4], [3, 0]]))
    ek, ev = kc.copy(), vc.copy()
    ek[4], ev[4] = kc[1], vc[1]
    ek[0], ev[0] = kc[3], vc[3]
    assert np.array_equal(k2, ek) and np.array_equal(v2, ev)


def check_storage_formats():
    """Known encodings: bf16 1.0 = 0x3F80, -2.0 = 0xC000, 0.1 = 0x3DCD (rounded
    up from 0x3DCCCCCD), 1 + 2^-8 ties to even 0x3F80, 1 + 3*2^-8 ties to
    0x3F82; fp16 1.0 = 0x3C00, 65504 = 0x7BFF, 2^-24 = 0x0001."""
    b = O.encode_bits(np.array([1.0, -2.0, 0.1, 1 + 2 ** -8, 1 + 3 * 2 ** -8]), O.BF16)
    assert b.tolist() == [0x3F80, 0xC000, 0x3DCD, 0x3F80, 0x3F82]
    assert O.decode_bits(np.array([0x3F80, 0xC000, 0x3DCD], np.uint16), O.BF16).tolist() == \
        [1.0, -2.0, 0.10009765625]
    h = O.encode_bits(np.array([1.0, 65504.0, 2.0 ** -24]), O.F16)
    assert h.tolist() == [0x3C00, 0x7BFF, 0x0001]
    assert O.decode_bits(h, O.F16).tolist() == [1.0, 65504.0, 2.0 ** -24]


ALL_CHECKS = [
    check_block_table_example,
    check_append_rule_example,
    check_generator_follows_append_rule,
    check_materialize_roundtrip,
    check_single_token_returns_value,
    check_two_token_sigmoid,
    check_uniform_weights_give_mean,
    check_dominant_key,
    check_against_torch_sdpa,
    check_gqa_grouping,
    check_brute_force_tiny,
    check_empty_sequence_is_zero,
    check_placement_invariance,
    check_table_padding_ignored,
    check_shared_prefix_equals_private_copy,
    check_split_lse_combine,
    check_reshape_and_cache_example,
    check_copy_blocks_example,
    check_storage_formats,
]


# ---------------------------------------------------------------------------
# 8-bit (E4M3) pools
# ---------------------------------------------------------------------------

def check_e4m3_known_codes():
    """Codes fixed by the format (1 sign, 4 exponent bits with bias 7, 3
    mantissa bits, subnormals m * 2^-9, largest finite 448, S.1111.111 NaN),
    round to nearest with ties to even, saturation to 448."""
    vals = np.array([1.0, -2.0, 448.0, 500.0, -1e9, 2.0 ** -9, 2.0 ** -6, 0.0, 1.0625, 1.1875,
                     1.5 * 2.0 ** -9, 0.9 * 2.0 ** -10, 240.0, 232.0])
    want = [0x38, 0xC0, 0x7E, 0x7E, 0xFE, 0x01, 0x08, 0x00, 0x38, 0x3A, 0x02, 0x00, 0x77, 0x76]
    assert O.e4m3_encode(vals).tolist() == want
    assert O.e4m3_decode(np.array([0x38, 0x7E, 0x01, 0x08, 0xB9], np.uint8)).tolist() == \
        [1.0, 448.0, 2.0 ** -9, 2.0 ** -6, -1.125]
    assert np.isnan(O.e4m3_decode(np.array([0x7F, 0xFF], np.uint8))).all()


def check_e4m3_all_codes_roundtrip():
    codes = np.arange(256, dtype=np.uint8)
    v = O.e4m3_decode(codes)
    fin = ~np.isnan(v)
    assert fin.sum() == 254
    assert np.array_equal(O.e4m3_encode(v[fin]), codes[fin])
    pos = np.sort(v[fin][v[fin] > 0])
    assert pos[0] == 2.0 ** -9 and pos[-1] == 448.0 and len(pos) == 126


def check_e4m3_against_torch():
    """Library special case: torch's float8_e4m3fn conversion (round to
    nearest even) agrees on in-range values."""
    import torch

    rng = np.random.default_rng(9)
    x = (rng.standard_normal(100000) * np.exp(rng.uniform(-9, 6, 100000))).astype(np.float32)
    x = x[np.abs(x) < 448]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(O.e4m3_encode(x.astype(np.float64)), ref)


def check_fp8_cache_write_example():
    """Two tokens into 8-token blocks: slot 3 and slot 13 (block 1, position 5);
    K lands in row (block, head, position), V in column (block, head, :, position)."""
    N, H, B, D = 3, 2, 8, 4
    kc = np.full((N, H, B, D), 0x7F, np.uint8)
    vc = np.full((N, H, D, B), 0x7F, np.uint8)
    one, two = 0x3C00, 0x4000  # fp16 1.0, 2.0
    key = np.array([[[one] * D] * H, [[two] * D] * H], np.uint16)
    value = key.copy()
    k2, v2 = O.reshape_and_cache_fp8(kc, vc, key, value, np.array([3, 13]), B, 0.5, 2.0, W.F16)
    # 1.0 / 0.5 = 2 -> 0x40; 2.0 / 0.5 = 4 -> 0x48; 1.0 / 2 = 0.5 -> 0x30; 2.0 / 2 = 1 -> 0x38
    ek, ev = kc.copy(), vc.copy()
    ek[0, :, 3, :] = 0x40
    ek[1, :, 5, :] = 0x48
    ev[0, :, :, 3] = 0x30
    ev[1, :, :, 5] = 0x38
    assert np.array_equal(k2, ek) and np.array_equal(v2, ev)


def check_fp8_decode_matches_fp16_decode():
    """With scales that are powers of two every E4M3 value is exact in fp16:
    decoding the 8-bit pools equals decoding fp16 pools that hold those
    values in the fp16 layout (pins the 8-bit layouts to the fp16 path)."""
    base = W.small_case(51, num_seqs=5, num_q_heads=8, num_kv_heads=2, head_dim=16, block_size=8,
                        dtype=W.F16, max_len=40, write_new_token=False)
    f8 = W.fp8_variant(base, 52, k_scale=0.25, v_scale=2.0)
    kv = O.e4m3_decode(f8.k_cache) * 0.25
    vv = O.e4m3_decode(f8.v_cache) * 2.0
    k16 = O.encode_bits(kv, W.F16)
    v16 = O.encode_bits(vv.transpose(0, 1, 3, 2), W.F16)
    ref = O.paged_attention_decode(base.q, k16, v16, base.block_tables, base.context_lens, 8, base.scale, W.F16)
    got = O.paged_attention_decode_fp8(base.q, f8.k_cache, f8.v_cache, base.block_tables, base.context_lens,
                                       8, base.scale, 0.25, 2.0, W.F16)
    assert np.array_equal(got, ref)


FP8_CHECKS = [
    check_e4m3_known_codes,
    check_e4m3_all_codes_roundtrip,
    check_e4m3_against_torch,
    check_fp8_cache_write_example,
    check_fp8_decode_matches_fp16_decode,
]
ALL_CHECKS += FP8_CHECKS


# ---------------------------------------------------------------------------
# Block manager: free pool, reference counts, append, copy-on-write, free
# ---------------------------------------------------------------------------

import oracle.block_manager as BMO  # noqa: E402


def check_manager_append_rule_example():
    """The append rule fixture, replayed through the manager: a request grows
    from 0 to 33 tokens one step at a time and then finishes."""
    fx = read_fixture(os.path.join(GOLDEN, "append_rule_example.txt"))
    B = fx["block_size"][0]
    m = BMO.BlockManager(16, B, 8, free_order=list(fx["free_pool"]))
    m.add_sequence(0, 0)
    slots = [m.append([0])[0][0] for _ in range(fx["tokens"][0])]
    assert m.tables[0] == fx["expect_table"]
    for t in (0, 15, 16, 31, 32):
        assert slots[t] == fx[f"expect_slot_token_{t}"][0], t
    m.free_sequence(0)
    assert list(m.free) == fx["expect_free_after_finish"]


def check_manager_copy_on_write_example():
    fx = read_fixture(os.path.join(GOLDEN, "copy_on_write_example.txt"))
    B, N = fx["block_size"][0], fx["num_blocks"][0]
    m = BMO.BlockManager(N, B, 8)
    m.add_sequence(9, fx["prompt_tokens"][0])
    assert m.tables[9] == fx["expect_prompt_table"]
    m.fork(9, 1)
    m.fork(9, 2)
    m.free_sequence(9)
    slots, copies = m.append([1, 2])
    assert slots == [fx["expect_slot_A"][0], fx["expect_slot_B"][0]]
    assert copies == [tuple(fx["expect_copy"])]
    assert m.tables[1] == fx["expect_table_A"] and m.tables[2] == fx["expect_table_B"]
    assert list(m.free) == fx["expect_free_after_step"]
    m.free_sequence(1)
    assert list(m.free) == fx["expect_free_after_A"]
    m.free_sequence(2)
    assert list(m.free) == fx["expect_free_after_B"]


def _paged_view(pool, table, length, B):
    return [pool.get(table[t // B] * B + t % B) for t in range(length)]


def check_manager_brute_force_churn():
    """Random arrivals, forks, decode steps and finishes against the plain
    logical model (each request is the list of its tokens).  After every
    operation: reading each request through its Block Table gives its tokens;
    every block's reference count is the number of tables that hold it;
    the free pool holds exactly the unreferenced blocks, once each; a step is
    refused exactly when the pool is short, and then changes nothing."""
    rng = np.random.default_rng(5)
    for trial in range(6):
        B = int(rng.choice([2, 4, 16]))
        N = int(rng.integers(6, 40))
        m = BMO.BlockManager(N, B, 64)
        pool: dict[int, int] = {}  # slot -> token value (the physical contents)
        hist: dict[int, list[int]] = {}  # request -> its tokens (the logical model)
        next_id, next_val = 0, 1
        for _ in range(150):
            op = rng.random()
            live = sorted(hist)
            if op < 0.2 or not live:
                n = int(rng.integers(0, 3 * B))
                if -(-n // B) <= len(m.free):
                    vals = list(range(next_val, next_val + n))
                    next_val += n
                    for slot, v in zip(m.add_sequence(next_id, n), vals):
                        pool[slot] = v
                    hist[next_id] = vals
                    next_id += 1
            elif op < 0.3:
                p = int(rng.choice(live))
                m.fork(p, next_id)
                hist[next_id] = list(hist[p])
                next_id += 1
            elif op < 0.45:
                s = int(rng.choice(live))
                m.free_sequence(s)
                del hist[s]
            else:
                k = int(rng.integers(1, len(live) + 1))
                ids = [int(x) for x in rng.permutation(live)[:k]]
                need = m.blocks_needed(ids)
                before = (list(m.free), list(m.ref), {s: list(t) for s, t in m.tables.items()}, dict(m.lens))
                if need > len(m.free):
                    try:
                        m.append(ids)
                        raise AssertionError("step should have been refused")
                    except BMO.OutOfBlocks:
                        pass
                    assert (list(m.free), list(m.ref), m.tables, m.lens) == before
                else:
                    free_before = len(m.free)
                    slots, copies = m.append(ids)
                    assert free_before - len(m.free) == need
                    for src, dst in copies:  # copies run before the writes
                        for o in range(B):
                            if src * B + o in pool:
                                pool[dst * B + o] = pool[src * B + o]
                    for s, slot in zip(ids, slots):
                        pool[slot] = next_val
                        hist[s].append(next_val)
                        next_val += 1
            # invariants
            counts = [0] * N
            for s, t in m.tables.items():
                assert len(t) == -(-m.lens[s] // B) and m.lens[s] == len(hist[s])
                assert _paged_view(pool, t, m.lens[s], B) == hist[s], (trial, s)
                for b in t:
                    counts[b] += 1
            assert counts == m.ref
            assert sorted(m.free) == [b for b in range(N) if counts[b] == 0]


def check_manager_append_matches_append_rule():
    """For requests that share nothing, the manager's slots are the append
    rule's slots (the pinned single-table function) with the same pool."""
    rng = np.random.default_rng(8)
    B, N = 4, 30
    order = [int(x) for x in rng.permutation(N)]
    m = BMO.BlockManager(N, B, 64, free_order=list(order))
    free = list(order)
    tables = {0: [], 1: []}
    lens = {0: 0, 1: 0}
    m.add_sequence(0, 0)
    m.add_sequence(1, 0)
    for step in range(25):
        ids = [0, 1] if step % 3 else [1, 0]
        slots, copies = m.append(ids)
        assert copies == []
        for s, slot in zip(ids, slots):
            assert slot == O.append_token(tables[s], lens[s], free, B)
            lens[s] += 1
    assert m.tables == tables and list(m.free) == free


BM_CHECKS = [
    check_manager_append_rule_example,
    check_manager_copy_on_write_example,
    check_manager_brute_force_churn,
    check_manager_append_matches_append_rule,
]
ALL_CHECKS += BM_CHECKS



# ---------------------------------------------------------------------------
# Chunked prefill: causal attention of a chunk of new tokens over the cache
# ---------------------------------------------------------------------------

import oracle.prefill as PO  # noqa: E402


def _prefill_case(seed=9, dtype=W.F16, B=8, lens=(1, 9, 30, 17, 64), chunks=(1, 9, 7, 1, 20)):
    b = W.prefill_batch(seed, dtype=dtype, num_q_heads=6, num_kv_heads=2, head_dim=16, block_size=B,
                        context_lens=list(lens), chunk_lens=list(chunks))
    kc, vc = O.reshape_and_cache(b.k_cache, b.v_cache, b.key, b.value, b.slot_mapping, B)
    return b, kc, vc


def check_prefill_is_a_sequence_of_decode_steps():
    """Token j of a chunk sits at position p = L - C + j and sees positions
    0..p: its row equals the (pinned) decode of that sequence cut at p + 1."""
    b, kc, vc = _prefill_case()
    out = PO.paged_prefill(b.q, kc, vc, b.block_tables, b.query_start, b.context_lens, b.block_size, b.scale,
                           b.dtype)
    for s in range(b.num_seqs):
        L, t0, t1 = int(b.context_lens[s]), int(b.query_start[s]), int(b.query_start[s + 1])
        for j in range(t1 - t0):
            p = L - (t1 - t0) + j
            ref = O.decode_sequence(b.q[t0 + j], kc, vc, b.block_tables[s], p + 1, b.block_size, b.scale, b.dtype)
            assert np.allclose(out[t0 + j], ref, rtol=0, atol=1e-12), (s, j)


def check_prefill_against_torch_sdpa_causal():
    """Library special case: a whole-prompt prefill is torch's causal SDPA,
    and a chunk is SDPA with the explicit mask key position <= query
    position, both in float64 on the materialised K/V."""
    import torch
    b, kc, vc = _prefill_case(seed=10, dtype=W.BF16, lens=(12, 40), chunks=(12, 15))
    out = PO.paged_prefill(b.q, kc, vc, b.block_tables, b.query_start, b.context_lens, b.block_size, b.scale,
                           b.dtype)
    Hq, Hkv = b.num_q_heads, b.num_kv_heads
    for s in range(b.num_seqs):
        L, t0, t1 = int(b.context_lens[s]), int(b.query_start[s]), int(b.query_start[s + 1])
        C = t1 - t0
        K = torch.from_numpy(O.decode_bits(O.materialize(kc, b.block_tables[s], L, b.block_size), b.dtype))
        V = torch.from_numpy(O.decode_bits(O.materialize(vc, b.block_tables[s], L, b.block_size), b.dtype))
        q = torch.from_numpy(O.decode_bits(b.q[t0:t1], b.dtype)).transpose(0, 1)  # [Hq, C, D]
        K = K.repeat_interleave(Hq // Hkv, dim=0)
        V = V.repeat_interleave(Hq // Hkv, dim=0)
        if C == L:
            ref = torch.nn.functional.scaled_dot_product_attention(q, K, V, is_causal=True, scale=b.scale)
        else:
            mask = torch.arange(L)[None, :] <= (L - C + torch.arange(C))[:, None]
            ref = torch.nn.functional.scaled_dot_product_attention(q, K, V, attn_mask=mask, scale=b.scale)
        assert np.allclose(out[t0:t1], ref.transpose(0, 1).numpy(), rtol=0, atol=1e-12), s


def check_prefill_brute_force_tiny():
    """Pure-Python loops: per query token, per head, a table lookup per key."""
    b, kc, vc = _prefill_case(seed=11, B=4, lens=(6, 9), chunks=(3, 9))
    out = PO.paged_prefill(b.q, kc, vc, b.block_tables, b.query_start, b.context_lens, b.block_size, b.scale,
                           b.dtype)
    Hq, Hkv, D, B = b.num_q_heads, b.num_kv_heads, b.head_dim, b.block_size
    for s in range(b.num_seqs):
        L, t0, t1 = int(b.context_lens[s]), int(b.query_start[s]), int(b.query_start[s + 1])
        for j in range(t1 - t0):
            p = L - (t1 - t0) + j
            for h in range(Hq):
                g = h * Hkv // Hq
                q = [float(x) for x in O.decode_bits(b.q[t0 + j, h], b.dtype)]
                zs, vs = [], []
                for i in range(p + 1):
                    blk = int(b.block_tables[s][i // B])
                    k = O.decode_bits(kc[blk, g, i % B], b.dtype)
                    zs.append(b.scale * sum(q[d] * float(k[d]) for d in range(D)))
                    vs.append(O.decode_bits(vc[blk, g, i % B], b.dtype))
                m = max(zs)
                w = [math.exp(z - m) for z in zs]
                ref = sum(wi * vi for wi, vi in zip(w, vs)) / sum(w)
                assert np.allclose(out[t0 + j, h], ref, rtol=0, atol=1e-12)


PREFILL_CHECKS = [
    check_prefill_is_a_sequence_of_decode_steps,
    check_prefill_against_torch_sdpa_causal,
    check_prefill_brute_force_tiny,
]
ALL_CHECKS += PREFILL_CHECKS
