"""A multi-step decode loop with requests arriving, forking, growing and
finishing, driven by the C++ block manager: every step runs the block
copies, the cache write and decode attention on the GPU, and the outputs are
compared with attention over each request's logical token history (no paging
at all), computed by the oracle in float64 (B200 only).

The loop follows the scheduler iteration of lshu.cn/news/11644, section
"整体架构": admit new requests while the pool has room (their prompts written
at once), give every running request one new token, release the blocks of
finished requests at once.
"""

import numpy as np
import pytest
import torch

import oracle as O
import paged_kv_cache_407_b200 as pkv
import workloads as W
from paged_kv_cache_407_b200.block_manager import BlockManager
from parity import bits, compare, status_tensor
from workloads.device import bits_to_tensor

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "these tests need a CUDA device"
    from paged_kv_cache_407_b200.build import build
    build()
    pkv.library()


@pytest.mark.parametrize("dtype,B,Hq,Hkv,D", [(W.F16, 16, 8, 2, 128), (W.BF16, 8, 4, 4, 64),
                                              (W.F16, 32, 16, 2, 128)])
def test_decode_loop_with_churn(dtype, B, Hq, Hkv, D):
    rng = np.random.default_rng(2024 + B)
    N, M = 96, 24  # pool blocks, Block Table entries per request
    scale = 1.0 / np.sqrt(D)
    bm = BlockManager(N, B, M)
    poison = W.POISON_BITS[dtype]
    k_cache = bits_to_tensor(np.full((N, Hkv, B, D), poison, np.uint16), dtype, "cuda")
    v_cache = bits_to_tensor(np.full((N, Hkv, B, D), poison, np.uint16), dtype, "cuda")
    hist_k: dict[int, list] = {}  # request -> its K rows [Hkv, D] (bits), the logical truth
    hist_v: dict[int, list] = {}
    st = status_tensor()
    next_id = 0
    copies_seen = 0

    def kv_rows(n):
        k = W.to_bits(rng.standard_normal((n, Hkv, D), dtype=np.float32), dtype)
        v = W.to_bits(rng.standard_normal((n, Hkv, D), dtype=np.float32), dtype)
        return k, v

    def write(slots, k, v):
        pkv.reshape_and_cache(bits_to_tensor(k, dtype, "cuda"), bits_to_tensor(v, dtype, "cuda"),
                              k_cache, v_cache, torch.from_numpy(np.asarray(slots, np.int64)).cuda(),
                              d_status=st)

    for step in range(40):
        # admit: new prompts, and forks of running requests (shared prefixes)
        for _ in range(int(rng.integers(0, 3))):
            live = sorted(hist_k)
            if live and rng.random() < 0.4:
                parent = int(rng.choice(live))
                bm.fork(parent, next_id)
                hist_k[next_id] = list(hist_k[parent])
                hist_v[next_id] = list(hist_v[parent])
                next_id += 1
                continue
            n = int(rng.integers(1, 5 * B))
            if -(-n // B) > bm.num_free_blocks - 4:
                continue
            slots = bm.add_sequence(next_id, n)
            k, v = kv_rows(n)
            write(slots, k, v)
            hist_k[next_id], hist_v[next_id] = list(k), list(v)
            next_id += 1
        # finish: some requests end; requests at the table limit end too
        for s in sorted(hist_k):
            if rng.random() < 0.08 or bm.context_len(s) >= B * M - 1:
                bm.free_sequence(s)
                del hist_k[s], hist_v[s]
        live = sorted(hist_k)
        while live and bm.blocks_needed(live) > bm.num_free_blocks:  # preempt the longest
            s = max(live, key=lambda x: len(hist_k[x]))
            bm.free_sequence(s)
            del hist_k[s], hist_v[s]
            live.remove(s)
        if not live:
            continue
        # one decode step: copies, then the new tokens' writes, then attention
        slots, copies = bm.append(live)
        copies_seen += len(copies)
        if len(copies):
            pkv.copy_blocks(k_cache, v_cache, torch.from_numpy(copies).cuda(), d_status=st)
        k, v = kv_rows(len(live))
        write(slots, k, v)
        for i, s in enumerate(live):
            hist_k[s].append(k[i])
            hist_v[s].append(v[i])
        tables, lens = bm.block_tables(live)
        q = W.to_bits(rng.standard_normal((len(live), Hq, D), dtype=np.float32), dtype)
        out = torch.empty((len(live), Hq, D), dtype=k_cache.dtype, device="cuda")
        pkv.paged_attention_decode(out, bits_to_tensor(q, dtype, "cuda"), k_cache, v_cache,
                                   torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda(),
                                   int(lens.max()), scale, d_status=st)
        torch.cuda.synchronize()
        ref = np.empty((len(live), Hq, D))
        for i, s in enumerate(live):
            K = O.decode_bits(np.stack(hist_k[s]), dtype)  # [L, Hkv, D]
            V = O.decode_bits(np.stack(hist_v[s]), dtype)
            qd = O.decode_bits(q[i], dtype)
            for g in range(Hkv):
                heads = [h for h in range(Hq) if O.kv_head_of(h, Hq, Hkv) == g]
                ref[i, heads] = O.attend(qd[heads], K[:, g], V[:, g], scale)
        compare(bits(out), ref, dtype, f"step {step}")
        if step % 8 == 7:  # the pool read through the tables is each request's history
            kc, vc = bits(k_cache), bits(v_cache)
            for i, s in enumerate(live):
                L = int(lens[i])
                assert np.array_equal(O.materialize(kc, tables[i], L, B).transpose(1, 0, 2),
                                      np.stack(hist_k[s])), (step, s)
                assert np.array_equal(O.materialize(vc, tables[i], L, B).transpose(1, 0, 2),
                                      np.stack(hist_v[s])), (step, s)
    assert int(st.item()) == 0
    assert copies_seen > 0, "the loop never exercised copy-on-write"
    bm.close()
