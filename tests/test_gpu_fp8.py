"""GPU parity of the 8-bit (E4M3) KV path against the oracle: quantising cache
writes bit for bit, decode attention over 8-bit pools within the attention
tolerance, block copies of 8-bit pools bit for bit (B200 only)."""

import numpy as np
import pytest
import torch

import oracle as O
import paged_kv_cache_407_b200 as pkv
import workloads as W
from parity import compare, status_tensor
from workloads.device import bits_to_tensor, upload_fp8

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "these tests need a CUDA device"
    from paged_kv_cache_407_b200.build import build
    build()
    pkv.library()


def _u8(t):
    return t.cpu().numpy()


def _fp8_step(f8, partition_size=0, d_status=None, write=True):
    db = upload_fp8(f8)
    if write and f8.num_tokens:
        pkv.reshape_and_cache_fp8(db.key, db.value, db.k_cache, db.v_cache, db.slot_mapping, f8.k_scale,
                                  f8.v_scale, d_status=d_status)
    pkv.paged_attention_decode_fp8(db.out, db.q, db.k_cache, db.v_cache, db.block_tables, db.context_lens,
                                   f8.max_context_len, f8.scale, f8.k_scale, f8.v_scale,
                                   partition_size=partition_size, d_status=d_status)
    torch.cuda.synchronize()
    return db


def _oracle_step(f8, write=True, seqs=None):
    kc, vc = f8.k_cache, f8.v_cache
    if write and f8.num_tokens:
        kc, vc = O.reshape_and_cache_fp8(kc, vc, f8.key, f8.value, f8.slot_mapping, f8.block_size, f8.k_scale,
                                         f8.v_scale, f8.dtype)
    out = O.paged_attention_decode_fp8(f8.q, kc, vc, f8.block_tables, f8.context_lens, f8.block_size,
                                       f8.scale, f8.k_scale, f8.v_scale, f8.dtype, seqs=seqs)
    return kc, vc, out


@pytest.mark.parametrize("dtype", [W.F16, W.BF16])
@pytest.mark.parametrize("B,Hkv", [(16, 4), (32, 8), (64, 2)])
@pytest.mark.parametrize("scales", [(0.05, 0.03), (0.002, 0.001), (40.0, 60.0)])
def test_fp8_cache_write_bit_exact(dtype, B, Hkv, scales):
    """Quantising write, including saturated (tiny scales) and subnormal
    (large scales) codes."""
    base = W.small_case(300 + B + Hkv, num_seqs=9, num_q_heads=Hkv, num_kv_heads=Hkv, head_dim=128,
                        block_size=B, dtype=dtype, max_len=3 * B + 5)
    f8 = W.fp8_variant(base, 7, k_scale=scales[0], v_scale=scales[1])
    db = upload_fp8(f8)
    st = status_tensor()
    pkv.reshape_and_cache_fp8(db.key, db.value, db.k_cache, db.v_cache, db.slot_mapping, f8.k_scale,
                              f8.v_scale, d_status=st)
    torch.cuda.synchronize()
    kc, vc = O.reshape_and_cache_fp8(f8.k_cache, f8.v_cache, f8.key, f8.value, f8.slot_mapping, B,
                                     f8.k_scale, f8.v_scale, dtype)
    assert np.array_equal(_u8(db.k_cache), kc)
    assert np.array_equal(_u8(db.v_cache), vc)
    assert int(st.item()) == 0


def test_fp8_cache_write_strided_and_unaligned_inputs():
    """Keys/values given as a slice of a fused QKV row (8-byte loads) and as
    rows that are only 2-byte aligned (element loads); padding slots skipped."""
    b = W.small_case(17, num_seqs=7, num_q_heads=4, num_kv_heads=4, head_dim=128, block_size=16,
                     dtype=W.F16, max_len=50)
    f8 = W.fp8_variant(b, 3, k_scale=0.09, v_scale=0.13)
    slots = b.slot_mapping.copy()
    slots[[2, 5]] = -1
    T, H, D = b.key.shape
    kc, vc = O.reshape_and_cache_fp8(f8.k_cache, f8.v_cache, b.key, b.value, slots, 16, f8.k_scale,
                                     f8.v_scale, b.dtype)
    s_dev = torch.from_numpy(slots).cuda()
    wide_k = np.zeros((T, 3, H, D), np.uint16)
    wide_v = np.zeros((T, 3, H, D), np.uint16)
    wide_k[:, 1], wide_v[:, 2] = b.key, b.value
    k_view = bits_to_tensor(wide_k, b.dtype, "cuda")[:, 1]
    v_view = bits_to_tensor(wide_v, b.dtype, "cuda")[:, 2]
    db = upload_fp8(f8)
    pkv.reshape_and_cache_fp8(k_view, v_view, db.k_cache, db.v_cache, s_dev, f8.k_scale, f8.v_scale)
    torch.cuda.synchronize()
    assert np.array_equal(_u8(db.k_cache), kc) and np.array_equal(_u8(db.v_cache), vc)
    flat_k = bits_to_tensor(np.concatenate([[0], b.key.ravel()]).astype(np.uint16), b.dtype, "cuda")
    flat_v = bits_to_tensor(np.concatenate([[0], b.value.ravel()]).astype(np.uint16), b.dtype, "cuda")
    k_odd, v_odd = flat_k[1:].view(T, H, D), flat_v[1:].view(T, H, D)
    assert k_odd.data_ptr() % 8 != 0
    db = upload_fp8(f8)
    pkv.reshape_and_cache_fp8(k_odd, v_odd, db.k_cache, db.v_cache, s_dev, f8.k_scale, f8.v_scale)
    torch.cuda.synchronize()
    assert np.array_equal(_u8(db.k_cache), kc) and np.array_equal(_u8(db.v_cache), vc)


FP8_CASES = [
    # dtype, B, Hq, Hkv, max_len, partition
    (W.F16, 16, 32, 8, 900, 0),
    (W.BF16, 16, 8, 8, 700, 0),
    (W.BF16, 32, 32, 8, 1500, 512),
    (W.F16, 32, 16, 2, 800, 64),
    (W.F16, 64, 8, 1, 600, 128),
    (W.BF16, 16, 32, 2, 500, 0),   # 16 query heads per kv head
    (W.BF16, 16, 4, 4, 1200, 16),  # one block per partition, merge kernel path
    # groups that are not powers of two
    (W.F16, 16, 12, 4, 900, 0),     # GQA 3: tokens on M, five idle head columns
    (W.BF16, 32, 28, 4, 1500, 512),  # GQA 7
    (W.F16, 64, 24, 2, 700, 64),    # GQA 12: query-rows form
]


@pytest.mark.parametrize("dtype,B,Hq,Hkv,max_len,P", FP8_CASES)
def test_fp8_decode_parity(dtype, B, Hq, Hkv, max_len, P):
    pre = W.small_case(400 + B + Hq + max_len, num_seqs=12, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=128,
                       block_size=B, dtype=dtype, max_len=max_len)
    base = W.small_case(400 + B + Hq + max_len, num_seqs=12, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=128,
                        block_size=B, dtype=dtype, max_len=max_len, partition_size=P,
                        lens=[1, B, B + 1, max_len, *list(pre.context_lens[4:])])
    f8 = W.fp8_variant(base, 11, k_scale=0.11, v_scale=0.07)
    st = status_tensor()
    db = _fp8_step(f8, partition_size=P, d_status=st)
    kc, vc, ref = _oracle_step(f8)
    assert np.array_equal(_u8(db.k_cache), kc) and np.array_equal(_u8(db.v_cache), vc)
    compare(db.out.view(torch.int16).cpu().numpy().view(np.uint16), ref, dtype,
            f"fp8 decode {dtype} B{B} {Hq}/{Hkv} P{P}")
    assert int(st.item()) == 0


def test_fp8_copy_blocks_bit_exact():
    base = W.prefix_share(19, num_seqs=9, prefix_tokens=70, suffix_range=(5, 40), num_q_heads=16,
                          num_kv_heads=4, head_dim=128, block_size=16, dtype=W.BF16)
    f8 = W.fp8_variant(base, 5)
    db = upload_fp8(f8)
    pkv.copy_blocks(db.k_cache, db.v_cache, db.cow_pairs)
    torch.cuda.synchronize()
    kc, vc = O.copy_blocks(f8.k_cache, f8.v_cache, base.cow_pairs)
    assert np.array_equal(_u8(db.k_cache), kc) and np.array_equal(_u8(db.v_cache), vc)


@pytest.mark.parametrize("dtype,B", [(W.F16, 16), (W.BF16, 32), (W.F16, 64)])
def test_fp8_decode_every_finite_code(dtype, B):
    """Pools whose codes cover all 254 finite E4M3 codes (subnormal, small and
    large exponent fields alike), not only the mid-range codes the other
    cases draw; scales keep the dequantised values O(1)."""
    base = W.small_case(470 + B, num_seqs=12, num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=B,
                        dtype=dtype, max_len=700, partition_size=0)
    f8 = W.fp8_variant(base, 13, k_scale=1.0 / 64.0, v_scale=1.0 / 448.0, full_range=True)
    seen = set()
    for s in range(base.num_seqs):
        L = int(base.context_lens[s])
        nb = -(-L // B)
        seen |= set(np.unique(f8.k_cache[base.block_tables[s, :nb]]).tolist())
        seen |= set(np.unique(f8.v_cache[base.block_tables[s, :nb]]).tolist())
    assert seen >= set(range(256)) - {0x7F, 0xFF}, "the pools do not hold every finite code"
    st = status_tensor()
    db = _fp8_step(f8, d_status=st)
    kc, vc, ref = _oracle_step(f8)
    assert np.array_equal(_u8(db.k_cache), kc) and np.array_equal(_u8(db.v_cache), vc)
    compare(db.out.view(torch.int16).cpu().numpy().view(np.uint16), ref, dtype,
            f"fp8 decode, every finite code, {dtype} B{B}")
    assert int(st.item()) == 0


# ------------------------------------------------ bench batches at full size
# The 8-bit variants of the decode batches that the benchmark times with
# --kv-dtype e4m3, built with the same seed (777) and run in the same launch
# configuration (the batch's own partition size: automatic, or 512 tokens for
# the long-context batch); the oracle computes a seeded sample of sequences.

def _fp8_bench_case(base, sample, where):
    f8 = W.fp8_variant(base, 777)
    st = status_tensor()
    db = _fp8_step(f8, partition_size=base.partition_size, d_status=st)
    assert int(st.item()) == 0
    kc, vc, ref = _oracle_step(f8, seqs=sample)
    assert np.array_equal(_u8(db.k_cache), kc) and np.array_equal(_u8(db.v_cache), vc)
    return compare(db.out.view(torch.int16).cpu().numpy().view(np.uint16), ref, base.dtype, where)


def test_fp8_llama7b_shaped_sampled():
    base = W.llama7b_mha()
    seqs = sorted(np.random.default_rng(2).choice(base.num_seqs, 6, replace=False).tolist())
    stats = _fp8_bench_case(base, seqs, "fp8 llama7b_mha (bench batch)")
    assert stats["literal_ok"]


def test_fp8_gqa_write_sampled():
    base = W.gqa_write()
    seqs = sorted(np.random.default_rng(3).choice(base.num_seqs, 24, replace=False).tolist())
    stats = _fp8_bench_case(base, seqs, "fp8 gqa_write (bench batch)")
    assert stats["combined_ok"]


def test_fp8_long_context_sampled():
    base = W.long_context()
    assert base.partition_size == 512
    stats = _fp8_bench_case(base, [0, 2], "fp8 long_context (bench batch)")
    assert stats["combined_ok"]
