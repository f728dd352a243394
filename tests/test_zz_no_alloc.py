"""The allocation-free decode entry point (pkv_paged_attention_decode_noalloc)
against the regular one, for callers that cannot allocate device memory: its
split-K scratch is the library's built-in buffer instead of a caller workspace.

Both entry points run the same kernels with the same plan on the same inputs,
so their outputs must agree bit for bit; any difference would be a leak of an
earlier call's contents from the shared buffer.  The cases cover every way a
call uses the scratch: no split (scratch unused), two partitions (arrival
counters cleared by an asynchronous memset), 3..32 partitions (counters cleared
by the planning kernel, merge inside the attention kernel) and more than 32
partitions (merge kernel).  They run back to back and then again, so each call
finds the buffer holding another call's partials.  B200 only; kept in the
last-collected file so a stop-at-first-failure run has already run every other
test."""

import pytest
import torch

import paged_kv_cache_407_b200 as pkv
import workloads as W
from paged_kv_cache_407_b200 import binding as bd
from parity import bits, compare, oracle_caches, oracle_out, status_tensor
from workloads.device import upload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "these tests need a CUDA device"
    from paged_kv_cache_407_b200.build import build
    build()
    pkv.library()


# name: (seed, small_case arguments, range of the partition count of the longest sequence)
CASES = {
    "no split": (310, dict(num_seqs=6, num_q_heads=8, num_kv_heads=2, head_dim=128, block_size=16,
                           dtype=W.F16, max_len=300, partition_size=512), (1, 1)),
    "two partitions": (311, dict(num_seqs=5, num_q_heads=16, num_kv_heads=4, head_dim=64, block_size=16,
                                 dtype=W.BF16, min_len=300, max_len=500, partition_size=256), (2, 2)),
    "planned split": (301, dict(num_seqs=9, num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=16,
                                dtype=W.BF16, max_len=1500, partition_size=128), (3, 32)),
    "merge kernel": (312, dict(num_seqs=2, num_q_heads=8, num_kv_heads=2, head_dim=64, block_size=16,
                               dtype=W.F16, max_len=8192, partition_size=128, lens=[8192, 8001]), (33, 64)),
}


def _prepared(seed, kw):
    b = W.small_case(seed, **kw)
    db = upload(b)
    pkv.reshape_and_cache(db.key, db.value, db.k_cache, db.v_cache, db.slot_mapping)
    return b, db


def _regular(b, db):
    out = torch.full_like(db.q, float("nan"))
    pkv.paged_attention_decode(out, db.q, db.k_cache, db.v_cache, db.block_tables, db.context_lens,
                               b.max_context_len, b.scale, partition_size=b.partition_size)
    return out


def _noalloc(b, db, st):
    out = torch.full_like(db.q, float("nan"))
    bd.paged_attention_decode_noalloc(out, db.q, db.k_cache, db.v_cache, db.block_tables, db.context_lens,
                                      b.max_context_len, b.scale, partition_size=b.partition_size, d_status=st)
    return out


def test_noalloc_matches_the_regular_entry_point_on_consecutive_calls():
    prepared = {}
    for name, (seed, kw, parts) in CASES.items():
        b, db = _prepared(seed, kw)
        P = b.partition_size
        nb = -(-b.max_context_len // b.block_size)
        assert parts[0] <= -(-nb // (P // b.block_size)) <= parts[1], name
        assert pkv.workspace_size(b.num_seqs, b.num_q_heads, b.num_kv_heads, b.head_dim, b.block_size,
                                  b.max_context_len, P) <= bd.NOALLOC_SCRATCH_BYTES
        prepared[name] = (b, db, _regular(b, db))
    torch.cuda.synchronize()
    st = status_tensor()
    # every case, then every case again: each call meets the buffer as another
    # call left it
    for rnd in range(2):
        for name, (b, db, ref) in prepared.items():
            got = _noalloc(b, db, st)
            torch.cuda.synchronize()
            assert int(st.item()) == 0, (name, rnd)
            assert torch.equal(got.view(torch.int16), ref.view(torch.int16)), \
                f"{name}, call {rnd + 1}: differs from the regular entry point"
    # and both agree with the oracle
    for name, (b, db, ref) in prepared.items():
        kc, vc = oracle_caches(b, cow=False)
        compare(bits(ref), oracle_out(b, kc, vc), b.dtype, f"noalloc case {name}")


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
    with pytest.raises(bd.PkvError, match="more than the built-in.*PKV_ERR_TOO_LARGE"):
        bd.paged_attention_decode_noalloc(torch.empty_like(q), q, cache, cache, tables, lens, 32768, 0.1,
                                          partition_size=256)
