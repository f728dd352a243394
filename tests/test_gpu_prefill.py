"""Paged (chunked) prefill attention on tcgen05 against the oracle (B200
only): chunks of new tokens are written to the cache, then attend causally
over their sequences' blocks; every output element is compared with the
float64 oracle."""

import numpy as np
import pytest
import torch

import oracle.prefill as PO
import oracle as O
import paged_kv_cache_407_b200 as pkv
import workloads as W
from parity import bits, compare, status_tensor
from workloads.device import upload_prefill

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "these tests need a CUDA device"
    from paged_kv_cache_407_b200.build import build
    build()
    pkv.library()


def _run(b, pad_rows=0):
    db = upload_prefill(b)
    st = status_tensor()
    if b.num_tokens:
        pkv.reshape_and_cache(db.key, db.value, db.k_cache, db.v_cache, db.slot_mapping, d_status=st)
    q = db.q
    out = torch.empty_like(q)
    if pad_rows:
        q = torch.cat([q, torch.zeros((pad_rows,) + tuple(q.shape[1:]), dtype=q.dtype, device=q.device)])
        out = torch.full_like(q, 3.0)
    pkv.paged_prefill(out, q, db.k_cache, db.v_cache, db.block_tables, db.query_start, db.context_lens,
                      b.max_query_len, b.scale, d_status=st)
    torch.cuda.synchronize()
    return out, int(st.item())


def _oracle(b):
    kc, vc = O.reshape_and_cache(b.k_cache, b.v_cache, b.key, b.value, b.slot_mapping, b.block_size)
    return PO.paged_prefill(b.q, kc, vc, b.block_tables, b.query_start, b.context_lens, b.block_size, b.scale,
                            b.dtype)


CASES = [
    # dtype, B, Hq, Hkv, context lengths, chunk lengths
    (W.F16, 16, 8, 8, [300, 129, 1, 200], [300, 40, 1, 77]),
    (W.BF16, 32, 32, 8, [700, 260], [200, 260]),
    (W.F16, 8, 16, 1, [333], [100]),
    (W.BF16, 64, 16, 8, [1000, 5, 70], [0, 5, 64]),
    (W.F16, 16, 4, 2, [128, 256, 129], [128, 128, 1]),
    (W.BF16, 16, 32, 4, [513, 90, 1000], [513, 17, 300]),  # 8 query heads per kv head: 16 tokens a tile
    (W.F16, 32, 16, 2, [64, 777], [64, 129]),
]


@pytest.mark.parametrize("dtype,B,Hq,Hkv,lens,chunks", CASES)
def test_prefill_parity(dtype, B, Hq, Hkv, lens, chunks):
    b = W.prefill_batch(900 + B + Hq, dtype=dtype, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=128, block_size=B,
                        context_lens=lens, chunk_lens=chunks)
    out, st = _run(b)
    assert st == 0
    compare(bits(out), _oracle(b), dtype, f"prefill {dtype} B{B} {Hq}/{Hkv}")


def test_rows_outside_every_chunk_are_not_written():
    b = W.prefill_batch(77, dtype=W.F16, num_q_heads=8, num_kv_heads=2, head_dim=128, block_size=16,
                        context_lens=[90, 40], chunk_lens=[30, 40])
    out, st = _run(b, pad_rows=5)
    assert st == 0
    tail = out[b.num_tokens:].float().cpu().numpy()
    assert np.all(tail == 3.0)
    compare(bits(out[: b.num_tokens].contiguous()), _oracle(b), W.F16, "prefill with padding rows")


def test_chunk_of_one_token_matches_decode():
    """A one-token chunk is a decode step: same result as the decode kernel
    within the tolerance of each against the oracle."""
    b = W.prefill_batch(78, dtype=W.BF16, num_q_heads=16, num_kv_heads=4, head_dim=128, block_size=16,
                        context_lens=[513, 64, 1000], chunk_lens=[1, 1, 1])
    out, st = _run(b)
    assert st == 0
    compare(bits(out), _oracle(b), W.BF16, "one-token chunks")


def test_bad_lengths_and_block_ids_are_flagged_not_faulted():
    """A sequence whose chunk is longer than its context is skipped with
    PKV_DEV_BAD_LEN (its rows untouched); a Block Table entry outside the
    pool raises PKV_DEV_BAD_BLOCK.  The other sequences are still exact."""
    b = W.prefill_batch(79, dtype=W.F16, num_q_heads=8, num_kv_heads=4, head_dim=128, block_size=16,
                        context_lens=[200, 150, 300], chunk_lens=[40, 50, 60])
    db = upload_prefill(b)
    st = status_tensor()
    pkv.reshape_and_cache(db.key, db.value, db.k_cache, db.v_cache, db.slot_mapping, d_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    lens = db.context_lens.clone()
    lens[1] = 20  # chunk of 50 tokens in a context of 20
    out = torch.full_like(db.q, 5.0)
    pkv.paged_prefill(out, db.q, db.k_cache, db.v_cache, db.block_tables, db.query_start, lens, b.max_query_len,
                      b.scale, d_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & pkv.DEV_BAD_LEN
    ref = _oracle(b)
    got = bits(out)
    for s in (0, 2):
        t0, t1 = int(b.query_start[s]), int(b.query_start[s + 1])
        compare(got[t0:t1], ref[t0:t1], W.F16, f"seq {s}")
    t0, t1 = int(b.query_start[1]), int(b.query_start[2])
    assert np.all(out[t0:t1].float().cpu().numpy() == 5.0)
    st.zero_()
    tables = db.block_tables.clone()
    tables[2, 3] = b.k_cache.shape[0] + 7
    pkv.paged_prefill(out, db.q, db.k_cache, db.v_cache, tables, db.query_start, db.context_lens, b.max_query_len,
                      b.scale, d_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & pkv.DEV_BAD_BLOCK
    got = bits(out)
    for s in (0, 1):
        t0, t1 = int(b.query_start[s]), int(b.query_start[s + 1])
        compare(got[t0:t1], ref[t0:t1], W.F16, f"seq {s}")


def test_long_chunks_sampled_rows_and_repeat_calls_bit_identical():
    """Many K/V tiles per query tile (up to 32): every role's pipeline wraps
    its stages and barrier phases many times.  Three calls on the same inputs
    give bit-identical outputs (a race between the tensor pipe and the
    softmax warps would show up as a difference), and sampled rows match the
    oracle."""
    b = W.prefill_batch(81, dtype=W.BF16, num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=16,
                        context_lens=[4096, 3000], chunk_lens=[1024, 3000])
    db = upload_prefill(b)
    st = status_tensor()
    pkv.reshape_and_cache(db.key, db.value, db.k_cache, db.v_cache, db.slot_mapping, d_status=st)
    outs = []
    for _ in range(3):
        out = torch.empty_like(db.q)
        pkv.paged_prefill(out, db.q, db.k_cache, db.v_cache, db.block_tables, db.query_start, db.context_lens,
                          b.max_query_len, b.scale, d_status=st)
        outs.append(out)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert all(torch.equal(outs[0], o) for o in outs[1:])
    kc, vc = O.reshape_and_cache(b.k_cache, b.v_cache, b.key, b.value, b.slot_mapping, b.block_size)
    rows = np.arange(0, b.num_tokens, 97)
    qs = np.asarray(b.query_start)
    Hq, Hkv = b.q.shape[1], kc.shape[1]
    ref = np.zeros((len(rows),) + b.q.shape[1:])
    mats = {}
    for i, t in enumerate(rows):
        s = int(np.searchsorted(qs, t, side="right") - 1)
        L, C = int(b.context_lens[s]), int(qs[s + 1] - qs[s])
        if s not in mats:
            mats[s] = (O.decode_bits(O.materialize(kc, b.block_tables[s], L, b.block_size), b.dtype),
                       O.decode_bits(O.materialize(vc, b.block_tables[s], L, b.block_size), b.dtype))
        K, V = mats[s]
        p = L - C + (t - qs[s])
        q = O.decode_bits(b.q[t], b.dtype)
        for g in range(Hkv):
            hs = [h for h in range(Hq) if O.kv_head_of(h, Hq, Hkv) == g]
            ref[i, hs] = O.attend(q[hs], K[g, : p + 1], V[g, : p + 1], b.scale)
    compare(bits(outs[0])[rows], ref, W.BF16, "long chunks, sampled rows")


def test_dynamic_and_static_item_orders_agree_bitwise():
    """The work items (query tile, kv head, sequence) taken from the item
    counter in the workspace, or in the fixed order without one: each item
    is computed whole by one CTA either way, so the outputs must agree bit
    for bit, on a batch whose chunks differ in length; and they match the
    oracle on sampled rows.  Two calls with the same workspace reuse its
    counter."""
    b = W.prefill_mixed()
    db = upload_prefill(b)
    st = status_tensor()
    pkv.reshape_and_cache(db.key, db.value, db.k_cache, db.v_cache, db.slot_mapping, d_status=st)
    ws = torch.full((pkv.PREFILL_WORKSPACE_BYTES,), 0xAB, dtype=torch.uint8, device="cuda")  # not zero: the call zeroes it
    outs = []
    for dynamic in (False, True, True):
        out = torch.full_like(db.q, float("nan"))
        pkv.paged_prefill(out, db.q, db.k_cache, db.v_cache, db.block_tables, db.query_start, db.context_lens,
                          b.max_query_len, b.scale, d_status=st, dynamic=dynamic, workspace=ws if dynamic else None)
        outs.append(out)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))
    assert torch.equal(outs[1].view(torch.int16), outs[2].view(torch.int16))
    kc, vc = O.reshape_and_cache(b.k_cache, b.v_cache, b.key, b.value, b.slot_mapping, b.block_size)
    qs = np.asarray(b.query_start)
    rows = np.arange(0, b.num_tokens, 211)
    Hq, Hkv = b.q.shape[1], kc.shape[1]
    ref = np.zeros((len(rows),) + b.q.shape[1:])
    for i, t in enumerate(rows):
        s = int(np.searchsorted(qs, t, side="right") - 1)
        L, C = int(b.context_lens[s]), int(qs[s + 1] - qs[s])
        K = O.decode_bits(O.materialize(kc, b.block_tables[s], L, b.block_size), b.dtype)
        V = O.decode_bits(O.materialize(vc, b.block_tables[s], L, b.block_size), b.dtype)
        p = L - C + (t - qs[s])
        q = O.decode_bits(b.q[t], b.dtype)
        for g in range(Hkv):
            hs = [h for h in range(Hq) if O.kv_head_of(h, Hq, Hkv) == g]
            ref[i, hs] = O.attend(q[hs], K[g, : p + 1], V[g, : p + 1], b.scale)
    compare(bits(outs[1])[rows], ref, b.dtype, "prefill mixed batch, dynamic order, sampled rows")


def test_one_long_context_short_chunk():
    """A 64-token chunk at the end of a 40000-token context (313 K/V tiles, the
    last one ragged) and a second sequence of 3 tokens: the load warps' block-id
    ring, the stage counters and every barrier phase wrap hundreds of times
    inside one item.  Every output element against the oracle."""
    b = W.prefill_batch(83, dtype=W.BF16, num_q_heads=8, num_kv_heads=2, head_dim=128, block_size=16,
                        context_lens=[40000, 3], chunk_lens=[64, 3])
    out, st = _run(b)
    assert st == 0
    compare(bits(out), _oracle(b), W.BF16, "prefill 40000-token context, 64-token chunk")


@pytest.mark.parametrize("name", sorted(W.PREFILL_WORKLOADS))
def test_bench_prefill_workloads_sampled_rows(name):
    """The bench's prefill batches at full size, in the launch the bench times:
    sampled rows (every 509th token, all heads) against the oracle, and no
    device status."""
    b = W.PREFILL_WORKLOADS[name]()
    db = upload_prefill(b)
    st = status_tensor()
    pkv.reshape_and_cache(db.key, db.value, db.k_cache, db.v_cache, db.slot_mapping, d_status=st)
    out = torch.empty_like(db.q)
    pkv.paged_prefill(out, db.q, db.k_cache, db.v_cache, db.block_tables, db.query_start, db.context_lens,
                      b.max_query_len, b.scale, d_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    kc, vc = O.reshape_and_cache(b.k_cache, b.v_cache, b.key, b.value, b.slot_mapping, b.block_size)
    rows = np.arange(0, b.num_tokens, 509)
    qs = np.asarray(b.query_start)
    Hq, Hkv = b.q.shape[1], kc.shape[1]
    ref = np.zeros((len(rows),) + b.q.shape[1:])
    for i, t in enumerate(rows):
        s = int(np.searchsorted(qs, t, side="right") - 1)
        L, C = int(b.context_lens[s]), int(qs[s + 1] - qs[s])
        p = L - C + (t - qs[s])
        K = O.decode_bits(O.materialize(kc, b.block_tables[s], p + 1, b.block_size), b.dtype)
        V = O.decode_bits(O.materialize(vc, b.block_tables[s], p + 1, b.block_size), b.dtype)
        q = O.decode_bits(b.q[t], b.dtype)
        for g in range(Hkv):
            hs = [h for h in range(Hq) if O.kv_head_of(h, Hq, Hkv) == g]
            ref[i, hs] = O.attend(q[hs], K[g], V[g], b.scale)
    compare(bits(out)[rows], ref, b.dtype, f"{name}, sampled rows")
