"""GPU parity of the three kernels against the oracle on small seeded batches
that span several tiles, partitions and a ragged tail (B200 only)."""

import numpy as np
import pytest
import torch

import oracle as O
import paged_kv_cache_407_b200 as pkv
import workloads as W
from parity import bits, compare, oracle_caches, oracle_out, run_step, status_tensor
from workloads.device import bits_to_tensor, upload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "these tests need a CUDA device"
    from paged_kv_cache_407_b200.build import build
    build()
    pkv.library()


# --------------------------------------------------------------- cache write
@pytest.mark.parametrize("dtype", [W.F16, W.BF16])
@pytest.mark.parametrize("B,D,Hkv", [(16, 64, 4), (8, 128, 2), (32, 128, 8), (64, 64, 1)])
def test_reshape_and_cache_bit_exact(dtype, B, D, Hkv):
    b = W.small_case(100 + B + D, num_seqs=9, num_q_heads=Hkv, num_kv_heads=Hkv, head_dim=D,
                     block_size=B, dtype=dtype, max_len=3 * B + 5)
    db = upload(b)
    st = status_tensor()
    pkv.reshape_and_cache(db.key, db.value, db.k_cache, db.v_cache, db.slot_mapping, d_status=st)
    torch.cuda.synchronize()
    kc, vc = O.reshape_and_cache(b.k_cache, b.v_cache, b.key, b.value, b.slot_mapping, B)
    assert np.array_equal(bits(db.k_cache), kc)
    assert np.array_equal(bits(db.v_cache), vc)
    assert int(st.item()) == 0


def test_reshape_and_cache_padding_strides_and_unaligned_rows():
    b = W.small_case(7, num_seqs=6, num_q_heads=4, num_kv_heads=4, head_dim=64, block_size=16,
                     dtype=W.BF16, max_len=40)
    slots = b.slot_mapping.copy()
    slots[[1, 4]] = -1  # padding tokens write nothing
    T, H, D = b.key.shape
    # keys/values as a strided view: token stride 3*H*D (e.g. a slice of fused QKV)
    wide_k = np.zeros((T, 3, H, D), np.uint16)
    wide_v = np.zeros((T, 3, H, D), np.uint16)
    wide_k[:, 1], wide_v[:, 2] = b.key, b.value
    db = upload(b)
    k_view = bits_to_tensor(wide_k, b.dtype, "cuda")[:, 1]
    v_view = bits_to_tensor(wide_v, b.dtype, "cuda")[:, 2]
    s_dev = torch.from_numpy(slots).cuda()
    pkv.reshape_and_cache(k_view, v_view, db.k_cache, db.v_cache, s_dev)
    torch.cuda.synchronize()
    kc, vc = O.reshape_and_cache(b.k_cache, b.v_cache, b.key, b.value, slots, 16)
    assert np.array_equal(bits(db.k_cache), kc) and np.array_equal(bits(db.v_cache), vc)
    # rows that are only 2-byte aligned take the element-wise path
    db = upload(b)
    flat_k = bits_to_tensor(np.concatenate([[0], b.key.ravel()]).astype(np.uint16), b.dtype, "cuda")
    flat_v = bits_to_tensor(np.concatenate([[0], b.value.ravel()]).astype(np.uint16), b.dtype, "cuda")
    k_odd = flat_k[1:].view(T, H, D)
    v_odd = flat_v[1:].view(T, H, D)
    assert k_odd.data_ptr() % 16 != 0
    pkv.reshape_and_cache(k_odd, v_odd, db.k_cache, db.v_cache, s_dev)
    torch.cuda.synchronize()
    assert np.array_equal(bits(db.k_cache), kc) and np.array_equal(bits(db.v_cache), vc)


def test_reshape_and_cache_flags_slot_outside_pool():
    b = W.small_case(8, num_seqs=3, num_q_heads=2, num_kv_heads=2, head_dim=64, block_size=16,
                     dtype=W.F16, max_len=20)
    slots = b.slot_mapping.copy()
    slots[0] = b.num_blocks * 16 + 3
    db = upload(b)
    st = status_tensor()
    pkv.reshape_and_cache(db.key, db.value, db.k_cache, db.v_cache, torch.from_numpy(slots).cuda(), d_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & pkv.DEV_BAD_SLOT
    slots[0] = -1  # the bad token is skipped, the rest written
    kc, vc = O.reshape_and_cache(b.k_cache, b.v_cache, b.key, b.value, slots, 16)
    assert np.array_equal(bits(db.k_cache), kc)


# ---------------------------------------------------------------- block copy
@pytest.mark.parametrize("dtype,B,D,Hkv", [(W.F16, 16, 128, 8), (W.BF16, 32, 64, 2), (W.F16, 8, 64, 1)])
def test_copy_blocks_bit_exact(dtype, B, D, Hkv):
    b = W.prefix_share(9, num_seqs=11, prefix_tokens=5 * B - 3, suffix_range=(4, 3 * B), num_q_heads=2 * Hkv,
                       num_kv_heads=Hkv, head_dim=D, block_size=B, dtype=dtype)
    db = upload(b)
    st = status_tensor()
    pkv.copy_blocks(db.k_cache, db.v_cache, db.cow_pairs, d_status=st)
    torch.cuda.synchronize()
    kc, vc = O.copy_blocks(b.k_cache, b.v_cache, b.cow_pairs)
    assert np.array_equal(bits(db.k_cache), kc) and np.array_equal(bits(db.v_cache), vc)
    assert int(st.item()) == 0


def test_copy_blocks_flags_pair_outside_pool():
    b = W.prefix_share(10, num_seqs=4, prefix_tokens=30, suffix_range=(4, 10), num_q_heads=2,
                       num_kv_heads=1, head_dim=64, block_size=16)
    pairs = b.cow_pairs.copy()
    pairs[2, 1] = b.num_blocks  # out of range: skipped and flagged
    db = upload(b)
    st = status_tensor()
    pkv.copy_blocks(db.k_cache, db.v_cache, torch.from_numpy(pairs).cuda(), d_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & pkv.DEV_BAD_BLOCK
    kc, vc = O.copy_blocks(b.k_cache, b.v_cache, np.delete(pairs, 2, axis=0))
    assert np.array_equal(bits(db.k_cache), kc) and np.array_equal(bits(db.v_cache), vc)


# ----------------------------------------------------------- decode attention
DECODE_CASES = [
    # dtype, D, B, Hq, Hkv, max_len, partition
    (W.F16, 64, 16, 4, 4, 70, 0),
    (W.F16, 128, 16, 8, 8, 700, 0),      # MHA, auto split (256)
    (W.BF16, 128, 16, 32, 8, 900, 0),    # GQA 4
    (W.BF16, 128, 16, 32, 8, 900, 64),   # many small partitions
    (W.F16, 128, 32, 16, 2, 1500, 512),  # GQA 8, 32-token blocks
    (W.BF16, 128, 8, 8, 4, 300, 0),      # 8-token blocks
    (W.F16, 64, 64, 4, 1, 500, 128),     # 64-token blocks, GQA 4
    (W.BF16, 64, 32, 32, 2, 400, 0),     # GQA 16 (rows 8..15 of the MMA)
    (W.F16, 128, 64, 32, 2, 700, 256),   # GQA 16, 64-token blocks
    (W.BF16, 128, 16, 2, 2, 1200, 16),   # one block per partition
    # groups that are not powers of two: rows G..15 of the MMA idle
    (W.F16, 128, 16, 12, 4, 600, 0),     # GQA 3
    (W.BF16, 128, 32, 28, 4, 900, 256),  # GQA 7
    (W.F16, 64, 16, 24, 2, 500, 64),     # GQA 12 (rows 8..11 of the second half)
    (W.BF16, 128, 8, 10, 2, 400, 0),     # GQA 5, 8-token blocks
]


@pytest.mark.parametrize("dtype,D,B,Hq,Hkv,max_len,P", DECODE_CASES)
def test_decode_parity(dtype, D, B, Hq, Hkv, max_len, P):
    b = W.small_case(200 + D + B + Hq + max_len, num_seqs=12, num_q_heads=Hq, num_kv_heads=Hkv,
                     head_dim=D, block_size=B, dtype=dtype, max_len=max_len, partition_size=P)
    # force the edge lengths in: 1 token, exactly one block, one block + 1
    b = W.small_case(200 + D + B + Hq + max_len, num_seqs=12, num_q_heads=Hq, num_kv_heads=Hkv,
                     head_dim=D, block_size=B, dtype=dtype, max_len=max_len, partition_size=P,
                     lens=[1, B, B + 1, max_len, *list(b.context_lens[4:])])
    st = status_tensor()
    db = run_step(b, d_status=st)
    kc, vc = oracle_caches(b)
    compare(bits(db.out), oracle_out(b, kc, vc), dtype, f"decode {dtype} D{D} B{B} {Hq}/{Hkv} P{P}")
    assert int(st.item()) == 0


def test_single_token_gives_its_value_exactly():
    b = W.small_case(5, num_seqs=4, num_q_heads=8, num_kv_heads=2, head_dim=128, block_size=16,
                     dtype=W.BF16, max_len=1, lens=[1, 1, 1, 1])
    db = run_step(b)
    kc, vc = oracle_caches(b)
    G = 4
    for s in range(4):
        v = O.materialize(vc, b.block_tables[s], 1, 16)  # [Hkv, 1, D]
        for h in range(8):
            assert np.array_equal(bits(db.out)[s, h], v[h // G, 0])


def test_empty_sequences_give_zero_rows():
    b = W.small_case(6, num_seqs=5, num_q_heads=4, num_kv_heads=4, head_dim=64, block_size=16,
                     dtype=W.F16, max_len=600, lens=[0, 600, 0, 17, 300], partition_size=64)
    db = run_step(b)
    out = bits(db.out)
    assert np.all(out[[0, 2]] == 0)
    kc, vc = oracle_caches(b)
    compare(out, oracle_out(b, kc, vc, seqs=[1, 3, 4]), W.F16, "empty rows")


def test_partition_size_does_not_change_the_result():
    b = W.small_case(12, num_seqs=8, num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=16,
                     dtype=W.BF16, max_len=2000, key_outlier_frac=0.01)
    kc, vc = oracle_caches(b)
    ref = oracle_out(b, kc, vc)
    outs = {}
    for P in (16, 64, 256, 512, 2048, 0):
        db = run_step(b, partition_size=P)
        compare(bits(db.out), ref, W.BF16, f"P={P}")
        outs[P] = O.decode_bits(bits(db.out), W.BF16)
    for P, o in outs.items():
        assert np.max(np.abs(o - outs[2048])) < 4e-3, P


def test_repeated_calls_are_bit_identical():
    """Split partitions merged by whichever partition arrives last, the
    separate merge kernel (> 32 partitions) and unsplit sequences: the same
    inputs give the same bits on every call."""
    b = W.small_case(21, num_seqs=9, num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=16,
                     dtype=W.F16, max_len=1200)
    db = run_step(b)
    for P in (0, 32, 256):
        outs = []
        for _ in range(4):
            pkv.paged_attention_decode(db.out, db.q, db.k_cache, db.v_cache, db.block_tables, db.context_lens,
                                       b.max_context_len, b.scale, partition_size=P)
            torch.cuda.synchronize()
            outs.append(bits(db.out).copy())
        assert all(np.array_equal(o, outs[0]) for o in outs), P
        assert not np.any((outs[0] & 0x7C00) == 0x7C00), "inf/nan in output"


def test_placement_and_padding_do_not_change_bits():
    """Moving every block elsewhere in the pool, and filling table padding
    with other blocks' ids, gives bit-identical outputs."""
    b = W.small_case(13, num_seqs=10, num_q_heads=16, num_kv_heads=4, head_dim=128, block_size=16,
                     dtype=W.F16, max_len=500, write_new_token=False)
    base = bits(run_step(b, write=False).out)
    rng = np.random.default_rng(14)
    perm = rng.permutation(b.num_blocks)
    k2 = np.empty_like(b.k_cache)
    v2 = np.empty_like(b.v_cache)
    k2[perm], v2[perm] = b.k_cache, b.v_cache
    t2 = np.where(b.block_tables >= 0, perm[np.maximum(b.block_tables, 0)], -1).astype(np.int32)
    pad = t2 < 0
    t2[pad] = rng.integers(0, b.num_blocks, size=int(pad.sum()))
    b2 = W.PagedBatch(**{**b.__dict__, "k_cache": k2, "v_cache": v2, "block_tables": t2})
    assert np.array_equal(bits(run_step(b2, write=False).out), base)


def test_shared_prefix_equals_private_copies_bitwise():
    b = W.prefix_share(15, num_seqs=12, prefix_tokens=160, suffix_range=(20, 200), num_q_heads=32,
                       num_kv_heads=8, head_dim=128, block_size=16, dtype=W.F16)
    db = upload(b)
    pkv.copy_blocks(db.k_cache, db.v_cache, db.cow_pairs)
    pkv.reshape_and_cache(db.key, db.value, db.k_cache, db.v_cache, db.slot_mapping)
    out_private = torch.empty_like(db.q)
    out_shared = torch.empty_like(db.q)
    pkv.paged_attention_decode(out_private, db.q, db.k_cache, db.v_cache, db.block_tables,
                               db.context_lens, b.max_context_len, b.scale)
    pkv.paged_attention_decode(out_shared, db.q, db.k_cache, db.v_cache, db.block_tables_before_cow,
                               db.context_lens, b.max_context_len, b.scale)
    torch.cuda.synchronize()
    assert torch.equal(out_private.view(torch.int16), out_shared.view(torch.int16))
    kc, vc = oracle_caches(b)
    compare(bits(out_private), oracle_out(b, kc, vc), W.F16, "prefix")


def test_bad_block_and_length_are_flagged_not_faulted():
    b = W.small_case(16, num_seqs=6, num_q_heads=8, num_kv_heads=2, head_dim=128, block_size=16,
                     dtype=W.BF16, max_len=300, lens=[40, 300, 33, 70, 1, 129])
    tables = b.block_tables.copy()
    tables[2, 0] = b.num_blocks + 7  # outside the pool
    tables[3, 1] = -5
    db = upload(b)
    st = status_tensor()
    pkv.reshape_and_cache(db.key, db.value, db.k_cache, db.v_cache, db.slot_mapping)
    pkv.paged_attention_decode(db.out, db.q, db.k_cache, db.v_cache, torch.from_numpy(tables).cuda(),
                               db.context_lens, b.max_context_len, b.scale, d_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & pkv.DEV_BAD_BLOCK
    kc, vc = oracle_caches(b)
    compare(bits(db.out), oracle_out(b, kc, vc, seqs=[0, 1, 4, 5]), W.BF16, "untouched sequences")
    # a context length above max_context_len is clamped and flagged
    st.zero_()
    lens = db.context_lens.clone()
    lens[0] = b.max_context_len + 40
    pkv.paged_attention_decode(db.out, db.q, db.k_cache, db.v_cache, db.block_tables, lens,
                               b.max_context_len, b.scale, d_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & pkv.DEV_BAD_LEN


def test_runs_on_a_side_stream():
    b = W.small_case(17, num_seqs=7, num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=16,
                     dtype=W.BF16, max_len=800)
    db = upload(b)
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        pkv.reshape_and_cache(db.key, db.value, db.k_cache, db.v_cache, db.slot_mapping)
        pkv.paged_attention_decode(db.out, db.q, db.k_cache, db.v_cache, db.block_tables, db.context_lens,
                                   b.max_context_len, b.scale)
    side.synchronize()
    kc, vc = oracle_caches(b)
    compare(bits(db.out), oracle_out(b, kc, vc), W.BF16, "side stream")


def test_prepared_calls_match_plain_calls():
    """A prepared call (arguments checked and marshalled once) reissued on
    the same buffers gives the plain call's result bit for bit, and reflects
    new contents of those buffers (here: a changed query)."""
    b = W.small_case(88, num_seqs=7, num_q_heads=16, num_kv_heads=4, head_dim=128, block_size=16,
                     dtype=W.BF16, max_len=1200, partition_size=256)
    db = upload(b)
    st = status_tensor()
    write = pkv.reshape_and_cache(db.key, db.value, db.k_cache, db.v_cache, db.slot_mapping, d_status=st,
                                  prepare=True)
    out = torch.empty_like(db.q)
    dec = pkv.paged_attention_decode(out, db.q, db.k_cache, db.v_cache, db.block_tables, db.context_lens,
                                     b.max_context_len, b.scale, partition_size=256, d_status=st, prepare=True)
    write()
    assert dec() is out
    ref = pkv.paged_attention_decode(torch.empty_like(db.q), db.q, db.k_cache, db.v_cache, db.block_tables,
                                     db.context_lens, b.max_context_len, b.scale, partition_size=256)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    db.q.mul_(0.5)
    dec()
    ref2 = pkv.paged_attention_decode(torch.empty_like(db.q), db.q, db.k_cache, db.v_cache, db.block_tables,
                                      db.context_lens, b.max_context_len, b.scale, partition_size=256)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref2.view(torch.int16))
    assert not torch.equal(ref.view(torch.int16), ref2.view(torch.int16))
