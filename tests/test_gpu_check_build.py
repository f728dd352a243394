"""The check build of the library (libpkv_check.so, compiled with PKV_CHECK)
on a B200: the cache write refuses a step whose slots repeat, and the block
copy refuses pairs whose destination repeats or is also a source, with
PKV_ERR_ALIAS and before anything is written (lshu.cn/news/11644,
"方案：页式内存管理": a token owns one position of one block; "内存共享": a
shared block is only read, and each copy makes a new private block).  Calls
that respect those rules give the oracle's pools bit for bit, as the regular
build does."""

import ctypes

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from paged_kv_cache_407_b200 import binding as bd
from parity import bits, status_tensor
from workloads.device import upload, upload_fp8

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    assert torch.cuda.is_available(), "these tests need a CUDA device"
    from paged_kv_cache_407_b200.build import build_check
    build_check()
    chk = bd.check_library()
    assert chk.pkv_check_build() == 1
    return chk


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _write(lib, db, slots, st):
    return lib.pkv_reshape_and_cache(_p(db.key), _p(db.value), db.key.stride(0), db.value.stride(0),
                                     _p(db.k_cache), _p(db.v_cache), bd.cache_desc(db.k_cache), _p(slots),
                                     slots.numel(), _p(st), _stream())


def _copy(lib, k_cache, v_cache, desc, pairs, st):
    return lib.pkv_copy_blocks(_p(k_cache), _p(v_cache), desc, _p(pairs), pairs.shape[0], _p(st), _stream())


def _batch(dtype=W.F16):
    return W.small_case(31, num_seqs=6, num_q_heads=8, num_kv_heads=2, head_dim=128, block_size=16,
                        dtype=dtype, max_len=200)


@pytest.mark.parametrize("dtype", [W.F16, W.BF16])
def test_repeated_slot_is_refused_before_any_write(lib, dtype):
    b = _batch(dtype)
    db = upload(b)
    st = status_tensor()
    slots = b.slot_mapping.copy()
    slots[3] = slots[1]
    k0, v0 = db.k_cache.clone(), db.v_cache.clone()
    assert _write(lib, db, torch.from_numpy(slots).cuda(), st) == bd.ERR_ALIAS
    torch.cuda.synchronize()
    assert torch.equal(db.k_cache.view(torch.int16), k0.view(torch.int16))
    assert torch.equal(db.v_cache.view(torch.int16), v0.view(torch.int16))
    assert int(st.item()) == 0


def test_unique_slots_with_repeated_padding_write_the_oracle_pools(lib):
    b = _batch()
    db = upload(b)
    st = status_tensor()
    slots = b.slot_mapping.copy()
    slots[0] = slots[4] = -1  # padding tokens may repeat: they write nothing
    assert _write(lib, db, torch.from_numpy(slots).cuda(), st) == bd.OK
    torch.cuda.synchronize()
    kc, vc = O.reshape_and_cache(b.k_cache, b.v_cache, b.key, b.value, slots, b.block_size)
    assert np.array_equal(bits(db.k_cache), kc) and np.array_equal(bits(db.v_cache), vc)
    assert int(st.item()) == 0


def test_repeated_slot_is_refused_by_the_8bit_write(lib):
    f8 = W.fp8_variant(_batch(W.BF16), 3, k_scale=0.1, v_scale=0.05)
    db = upload_fp8(f8)
    st = status_tensor()
    k0, v0 = db.k_cache.clone(), db.v_cache.clone()
    desc = bd.fp8_cache_desc(db.k_cache, db.v_cache)

    def write(slots):
        return lib.pkv_reshape_and_cache_fp8(_p(db.key), _p(db.value), db.key.stride(0), db.value.stride(0),
                                             bd.PKV_BF16, _p(db.k_cache), _p(db.v_cache), desc, _p(slots),
                                             slots.numel(), ctypes.c_float(f8.k_scale), ctypes.c_float(f8.v_scale),
                                             _p(st), _stream())

    slots = f8.slot_mapping.copy()
    slots[5] = slots[2]
    assert write(torch.from_numpy(slots).cuda()) == bd.ERR_ALIAS
    torch.cuda.synchronize()
    assert torch.equal(db.k_cache, k0) and torch.equal(db.v_cache, v0)
    assert write(torch.from_numpy(f8.slot_mapping).cuda()) == bd.OK
    torch.cuda.synchronize()
    kc, vc = O.reshape_and_cache_fp8(f8.k_cache, f8.v_cache, f8.key, f8.value, f8.slot_mapping, f8.block_size,
                                     f8.k_scale, f8.v_scale, f8.dtype)
    assert np.array_equal(db.k_cache.cpu().numpy(), kc) and np.array_equal(db.v_cache.cpu().numpy(), vc)
    assert int(st.item()) == 0


def _prefix():
    return W.prefix_share(21, num_seqs=5, prefix_tokens=64, suffix_range=(4, 20), num_q_heads=4,
                          num_kv_heads=2, head_dim=64, block_size=16)


@pytest.mark.parametrize("case", ["dst twice", "dst is another pair's src", "dst is its own src"])
def test_overlapping_copy_pairs_are_refused_before_any_copy(lib, case):
    b = _prefix()
    db = upload(b)
    st = status_tensor()
    pairs = b.cow_pairs.copy()
    assert pairs.shape[0] >= 3
    if case == "dst twice":
        pairs[2, 1] = pairs[0, 1]
    elif case == "dst is another pair's src":
        pairs[1, 1] = pairs[0, 0]
    else:
        pairs[2, 1] = pairs[2, 0]
    k0, v0 = db.k_cache.clone(), db.v_cache.clone()
    assert _copy(lib, db.k_cache, db.v_cache, bd.cache_desc(db.k_cache), torch.from_numpy(pairs).cuda(),
                 st) == bd.ERR_ALIAS
    torch.cuda.synchronize()
    assert torch.equal(db.k_cache.view(torch.int16), k0.view(torch.int16))
    assert torch.equal(db.v_cache.view(torch.int16), v0.view(torch.int16))


def test_disjoint_copy_pairs_match_the_oracle(lib):
    """Every pair of the shared-prefix step reads the same shared block (a
    source may repeat); a pair outside the pool is skipped by the kernel and
    left out of the check, even where its dst repeats a valid one."""
    b = _prefix()
    db = upload(b)
    st = status_tensor()
    pairs = np.concatenate([b.cow_pairs, [[b.num_blocks + 3, b.cow_pairs[0, 1]]]]).astype(np.int64)
    assert len(set(b.cow_pairs[:, 0].tolist())) < b.cow_pairs.shape[0]
    assert _copy(lib, db.k_cache, db.v_cache, bd.cache_desc(db.k_cache), torch.from_numpy(pairs).cuda(),
                 st) == bd.OK
    torch.cuda.synchronize()
    assert int(st.item()) & bd.DEV_BAD_BLOCK
    kc, vc = O.copy_blocks(b.k_cache, b.v_cache, b.cow_pairs)
    assert np.array_equal(bits(db.k_cache), kc) and np.array_equal(bits(db.v_cache), vc)


def test_the_regular_build_is_not_the_check_build(lib):
    assert bd.library().pkv_check_build() == 0
