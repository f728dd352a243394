"""The allocation-free decode entry point (pkv_paged_attention_decode_noalloc)
against the regular one, for callers that cannot allocate device memory: its
split-K scratch is the library's built-in buffer instead of a caller workspace.
B200 only; kept in the last-collected file so a stop-at-first-failure run has
already run every other test."""

import numpy as np
import pytest
import torch

import oracle as O
import paged_kv_cache_407_b200 as pkv
import workloads as W
from paged_kv_cache_407_b200 import binding as bd
from parity import ATOL, RTOL, bits, status_tensor
from workloads.device import upload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "these tests need a CUDA device"
    from paged_kv_cache_407_b200.build import build
    build()
    pkv.library()


def _prepared(seed, **kw):
    b = W.small_case(seed, **kw)
    db = upload(b)
    pkv.reshape_and_cache(db.key, db.value, db.k_cache, db.v_cache, db.slot_mapping)
    return b, db


def _regular(b, db):
    out = torch.empty_like(db.q)
    pkv.paged_attention_decode(out, db.q, db.k_cache, db.v_cache, db.block_tables, db.context_lens,
                               b.max_context_len, b.scale, partition_size=b.partition_size)
    return out


def _noalloc(b, db, st):
    out = torch.full_like(db.q, float("nan"))
    bd.paged_attention_decode_noalloc(out, db.q, db.k_cache, db.v_cache, db.block_tables, db.context_lens,
                                      b.max_context_len, b.scale, partition_size=b.partition_size, d_status=st)
    return out


def _assert_close(got, ref, dtype):
    g = O.decode_bits(bits(got), dtype)
    r = O.decode_bits(bits(ref), dtype)
    assert np.all(np.abs(g - r) <= ATOL + RTOL * np.abs(r)), np.abs(g - r).max()


def test_noalloc_matches_the_regular_entry_point_on_consecutive_calls():
    # Two different batches that both need split-K scratch, then the first
    # again: the buffer keeps the previous call's partials and must not leak them.
    a, da = _prepared(301, num_seqs=9, num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=16,
                      dtype=W.BF16, max_len=1500, partition_size=128)
    b, dbb = _prepared(302, num_seqs=5, num_q_heads=16, num_kv_heads=16, head_dim=64, block_size=32,
                       dtype=W.F16, max_len=3000, partition_size=256)
    assert pkv.workspace_size(a.num_seqs, 32, 8, 128, 16, a.max_context_len, 128) > 0
    assert pkv.workspace_size(b.num_seqs, 16, 16, 64, 32, b.max_context_len, 256) > 0
    ref_a, ref_b = _regular(a, da), _regular(b, dbb)
    st = status_tensor()
    first = _noalloc(a, da, st)
    second = _noalloc(b, dbb, st)
    third = _noalloc(a, da, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    _assert_close(first, ref_a, W.BF16)
    _assert_close(second, ref_b, W.F16)
    _assert_close(third, ref_a, W.BF16)


def test_noalloc_refuses_sizes_beyond_its_buffer():
    # 64 sequences x 32 heads, 32768 tokens in 256-token partitions need
    # 64*32*128*130*4 bytes (136 MB) of partials: more than the buffer holds.
    S, Hq, D = 64, 32, 128
    need = pkv.workspace_size(S, Hq, 32, D, 16, 32768, 256)
    assert need > bd.NOALLOC_SCRATCH_BYTES
    q = torch.zeros(S, Hq, D, dtype=torch.float16, device="cuda")
    cache = torch.zeros(8, 32, 16, D, dtype=torch.float16, device="cuda")
    tables = torch.zeros(S, 2048, dtype=torch.int32, device="cuda")
    lens = torch.ones(S, dtype=torch.int32, device="cuda")
    with pytest.raises(bd.PkvError, match="PKV_ERR_TOO_LARGE"):
        bd.paged_attention_decode_noalloc(torch.empty_like(q), q, cache, cache, tables, lens, 32768, 0.1,
                                          partition_size=256)
