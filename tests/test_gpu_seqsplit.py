"""Decode with sequences split across GPUs, on one B200: the ranks' shares
are computed one after another by independent calls (no kernel waits on
another), stacked as the all-gather would stack them, and merged.  Checks
the attention state of one share against the oracle (fp32 output and
log-sum-exp) and the merged result against attention over whole sequences."""

import numpy as np
import pytest
import torch

import oracle as O
import paged_kv_cache_407_b200 as pkv
import workloads as W
from parity import bits, compare, status_tensor
from paged_kv_cache_407_b200.seqsplit import shard_tables
from workloads.device import upload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "these tests need a CUDA device"
    from paged_kv_cache_407_b200.build import build
    build()
    pkv.library()


def _written(b):
    db = upload(b)
    pkv.reshape_and_cache(db.key, db.value, db.k_cache, db.v_cache, db.slot_mapping)
    kc, vc = O.reshape_and_cache(b.k_cache, b.v_cache, b.key, b.value, b.slot_mapping, b.block_size)
    return db, kc, vc


def _oracle_state(b, kc, vc, tables, lens):
    S, Hq, D = b.q.shape
    Hkv = kc.shape[1]
    o = np.zeros((S, Hq, D))
    lse = np.full((S, Hq), -np.inf)
    for s in range(S):
        q = O.decode_bits(b.q[s], b.dtype)
        K = O.decode_bits(O.materialize(kc, tables[s], int(lens[s]), b.block_size), b.dtype)
        V = O.decode_bits(O.materialize(vc, tables[s], int(lens[s]), b.block_size), b.dtype)
        for h in range(Hq):
            m, l, on = O.partial_state(q[h:h + 1], K[O.kv_head_of(h, Hq, Hkv)],
                                       V[O.kv_head_of(h, Hq, Hkv)], b.scale)
            if l[0] > 0:
                o[s, h], lse[s, h] = on[0] / l[0], m[0] + np.log(l[0])
    return o, lse


CASES = [
    # dtype, B, Hq, Hkv, D, lens, partition
    (W.BF16, 32, 32, 8, 128, [5000, 3000, 33, 1], 512),
    (W.F16, 16, 8, 8, 64, [700, 16, 17, 0, 250], 0),
    (W.F16, 16, 16, 1, 128, [2100, 900], 64),
]


@pytest.mark.parametrize("dtype,B,Hq,Hkv,D,lens,P", CASES)
def test_share_state_matches_oracle(dtype, B, Hq, Hkv, D, lens, P):
    b = W.small_case(51 + B + Hq, num_seqs=len(lens), num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                     block_size=B, dtype=dtype, max_len=max(lens), lens=lens, key_outlier_frac=0.01)
    db, kc, vc = _written(b)
    tab, ln = shard_tables(b.block_tables, b.context_lens, B, 1, 3)
    S = b.num_seqs
    state = pkv.state_buffer(S * Hq, D, 1)[0]
    o, lse = pkv.state_views(state, S, Hq, D)
    st = status_tensor()
    pkv.paged_attention_decode_lse(o, lse, db.q, db.k_cache, db.v_cache, torch.from_numpy(tab).cuda(),
                                   torch.from_numpy(ln).cuda(), int(max(1, ln.max())), b.scale,
                                   partition_size=P, d_status=st)
    torch.cuda.synchronize()
    ro, rl = _oracle_state(b, kc, vc, tab, ln)
    got_o, got_l = o.double().cpu().numpy(), lse.double().cpu().numpy()
    assert np.all(np.abs(got_o - ro) <= 2e-3 + 1e-2 * np.abs(ro))
    live = np.isfinite(rl)
    assert np.array_equal(np.isfinite(got_l), live) and np.all(got_o[~live] == 0)
    assert np.max(np.abs(got_l[live] - rl[live])) < 2e-3
    assert int(st.item()) == 0


@pytest.mark.parametrize("dtype,B,Hq,Hkv,D,lens,P", CASES)
@pytest.mark.parametrize("world", [1, 2, 5])
def test_split_and_merge_equals_whole_sequence(dtype, B, Hq, Hkv, D, lens, P, world):
    b = W.small_case(61 + B + Hq, num_seqs=len(lens), num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                     block_size=B, dtype=dtype, max_len=max(lens), lens=lens, key_outlier_frac=0.01)
    db, kc, vc = _written(b)
    S = b.num_seqs
    states = pkv.state_buffer(S * Hq, D, world)  # what the all-gather delivers
    for r in range(world):
        tab, ln = shard_tables(b.block_tables, b.context_lens, B, r, world)
        o, lse = pkv.state_views(states[r], S, Hq, D)
        pkv.paged_attention_decode_lse(o, lse, db.q, db.k_cache, db.v_cache, torch.from_numpy(tab).cuda(),
                                       torch.from_numpy(ln).cuda(), int(max(1, ln.max())), b.scale,
                                       partition_size=P)
    out = torch.empty_like(db.q)
    pkv.merge_attention_states(out, states)
    torch.cuda.synchronize()
    ref = O.paged_attention_decode(b.q, kc, vc, b.block_tables, b.context_lens, B, b.scale, dtype)
    compare(bits(out), ref, dtype, f"split over {world}")
    zero = np.asarray(lens) == 0
    assert np.all(bits(out)[zero] == 0)


def test_merge_of_no_states_is_zero():
    out = torch.full((3, 4, 64), 7.0, dtype=torch.float16, device="cuda")
    pkv.merge_attention_states(out, torch.empty((0, 3 * 4 * 65), dtype=torch.float32, device="cuda"))
    torch.cuda.synchronize()
    assert torch.count_nonzero(out).item() == 0
