"""The failure path of the decode kernel's bounded waits, made to run on the GPU
without a fault: one TMA load is withheld, so its barrier never completes, and
every wait is limited to a few milliseconds.  The kernel must give up on that
wait, raise PKV_DEV_TIMEOUT, drain its other copies and exit; the rest of the
batch is computed normally and the device stays usable (B200 only)."""

import time

import pytest
import torch

import paged_kv_cache_407_b200 as pkv
import workloads as W
from paged_kv_cache_407_b200 import binding as bd
from parity import bits, compare, oracle_caches, oracle_out, run_step, status_tensor
from workloads.device import upload

pytestmark = pytest.mark.gpu

WAIT_US = 3000  # 3 ms per wait instead of about one second
PART = 512      # one partition per sequence (every length below is < 512)


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "these tests need a CUDA device"
    from paged_kv_cache_407_b200.build import build
    build()
    pkv.library()


def _batch():
    # 4 sequences of 160..400 tokens (10..25 blocks of 16), 8 q / 2 kv heads,
    # one partition per sequence
    return W.small_case(91, num_seqs=4, num_q_heads=8, num_kv_heads=2, head_dim=128, block_size=16,
                        dtype=W.F16, min_len=160, max_len=400)


@pytest.mark.parametrize("withheld", [0, 5, 9])
def test_withheld_load_ends_in_timeout_and_spares_the_rest(withheld):
    b = _batch()
    assert b.max_context_len <= PART
    assert withheld < -(-int(b.context_lens[0]) // 16)
    db = upload(b)
    pkv.reshape_and_cache(db.key, db.value, db.k_cache, db.v_cache, db.slot_mapping)
    torch.cuda.synchronize()
    st = status_tensor()
    out = torch.full_like(db.q, float("nan"))
    t0 = time.perf_counter()
    bd.test_decode_withheld_load(out, db.q, db.k_cache, db.v_cache, db.block_tables, db.context_lens,
                                 b.max_context_len, b.scale, withheld, WAIT_US, partition_size=PART, d_status=st)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert int(st.item()) == pkv.DEV_TIMEOUT, int(st.item())
    assert WAIT_US * 1e-6 <= elapsed < 0.5, elapsed  # waited out its limit, then returned
    # every row outside sequence 0's kv head 0 is the normal result
    kc, vc = oracle_caches(b, cow=False)
    ref = oracle_out(b, kc, vc)
    G = b.num_q_heads // b.num_kv_heads
    got = bits(out)
    compare(got[1:], ref[1:], b.dtype, f"withheld block {withheld}: other sequences")
    compare(got[0, G:], ref[0, G:], b.dtype, f"withheld block {withheld}: sequence 0, other kv heads")


def test_device_usable_after_a_timeout():
    b = _batch()
    db = upload(b)
    pkv.reshape_and_cache(db.key, db.value, db.k_cache, db.v_cache, db.slot_mapping)
    st = status_tensor()
    bd.test_decode_withheld_load(torch.empty_like(db.q), db.q, db.k_cache, db.v_cache, db.block_tables,
                                 db.context_lens, b.max_context_len, b.scale, 3, WAIT_US, partition_size=PART,
                                 d_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == pkv.DEV_TIMEOUT
    # a normal decode step right after, on a fresh status word, is exact again
    st2 = status_tensor()
    db2 = run_step(b, d_status=st2)
    assert int(st2.item()) == 0
    kc, vc = oracle_caches(b, cow=False)
    compare(bits(db2.out), oracle_out(b, kc, vc), b.dtype, "decode after a timeout")


def test_withheld_load_argument_checks():
    b = _batch()
    db = upload(b)
    out = torch.empty_like(db.q)
    args = (out, db.q, db.k_cache, db.v_cache, db.block_tables, db.context_lens, b.max_context_len, b.scale)
    with pytest.raises(bd.PkvError, match="PKV_ERR_BAD_SHAPE"):
        bd.test_decode_withheld_load(*args, 0, 0)           # a wait limit of 0
    with pytest.raises(bd.PkvError, match="PKV_ERR_BAD_PARTITION"):
        bd.test_decode_withheld_load(*args, 40, WAIT_US, partition_size=256)  # past the first partition
