"""A decode step captured once in a CUDA graph and replayed (B200 only): the
cache write of the step's new tokens and split-K decode attention are launched
from the graph, and between replays the step's inputs (new K/V rows, queries,
slots, lengths) are copied into the buffers the graph was captured on — the
way a serving loop removes the launch cost of small steps.  The graph is
captured with the Block Tables' capacity as max_context_len, so one graph
serves every step while the sequences grow.  Each replay is compared with the
oracle's attention over every sequence's logical history (no paging at all).

Cases: three partitions at the capacity (the planning kernel clears the split
counters) and two (an asynchronous memset does, captured as a graph node).  A
chunked prefill of a mixed batch is captured and replayed too (its item
counter reset is a memset node)."""

import numpy as np
import pytest
import torch

import oracle as O
import paged_kv_cache_407_b200 as pkv
import workloads as W
from parity import bits, compare, status_tensor
from workloads.device import bits_to_tensor

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "these tests need a CUDA device"
    from paged_kv_cache_407_b200.build import build
    build()
    pkv.library()


TORCH_DTYPE = {W.F16: torch.float16, W.BF16: torch.bfloat16}

CASES = [
    # dtype, B, Hq, Hkv, D, prompt lengths, partition tokens, replayed steps
    (W.F16, 16, 8, 2, 128, [100, 300, 700, 33], 256, 4),
    (W.BF16, 16, 16, 4, 128, [300, 450, 17], 256, 3),
]


@pytest.mark.parametrize("dtype,B,Hq,Hkv,D,lens,P,steps", CASES)
def test_decode_step_replayed_from_a_cuda_graph(dtype, B, Hq, Hkv, D, lens, P, steps):
    rng = np.random.default_rng(4100 + Hq + len(lens))
    S = len(lens)
    M = -(-(max(lens) + steps + 1) // B) + 1  # Block Table entries per sequence
    cap = M * B                                # max_context_len the graph is captured with
    N = S * M + 8
    tables_np = rng.permutation(N)[: S * M].reshape(S, M).astype(np.int32)
    scale = 1.0 / np.sqrt(D)
    poison = W.POISON_BITS[dtype]
    k_cache = bits_to_tensor(np.full((N, Hkv, B, D), poison, np.uint16), dtype, "cuda")
    v_cache = bits_to_tensor(np.full((N, Hkv, B, D), poison, np.uint16), dtype, "cuda")
    st = status_tensor()
    hist_k = [[] for _ in range(S)]  # per sequence: K rows [Hkv, D] (bits), the logical truth
    hist_v = [[] for _ in range(S)]

    def rows(n):
        return (W.to_bits(rng.standard_normal((n, Hkv, D), dtype=np.float32), dtype),
                W.to_bits(rng.standard_normal((n, Hkv, D), dtype=np.float32), dtype))

    def slot(s, t):
        return int(tables_np[s, t // B]) * B + t % B

    # prompts, written eagerly
    for s, L in enumerate(lens):
        k, v = rows(L)
        pkv.reshape_and_cache(bits_to_tensor(k, dtype, "cuda"), bits_to_tensor(v, dtype, "cuda"), k_cache, v_cache,
                              torch.tensor([slot(s, t) for t in range(L)], dtype=torch.int64, device="cuda"),
                              d_status=st)
        hist_k[s].extend(k)
        hist_v[s].extend(v)

    # the buffers the graph is captured on
    td = TORCH_DTYPE[dtype]
    new_k = torch.empty(S, Hkv, D, dtype=td, device="cuda")
    new_v = torch.empty_like(new_k)
    slots_t = torch.empty(S, dtype=torch.int64, device="cuda")
    q_t = torch.empty(S, Hq, D, dtype=td, device="cuda")
    ctx_t = torch.empty(S, dtype=torch.int32, device="cuda")
    tables_t = torch.from_numpy(tables_np).cuda()
    out_t = torch.empty_like(q_t)
    ws = torch.empty(max(16, pkv.workspace_size(S, Hq, Hkv, D, B, cap, P)), dtype=torch.uint8, device="cuda")

    def stage():
        """One new token per sequence into the captured buffers; returns the
        query bits of the step."""
        k, v = rows(S)
        q = W.to_bits(rng.standard_normal((S, Hq, D), dtype=np.float32), dtype)
        sl = [slot(s, len(hist_k[s])) for s in range(S)]
        for s in range(S):
            hist_k[s].append(k[s])
            hist_v[s].append(v[s])
        new_k.copy_(bits_to_tensor(k, dtype, "cuda"))
        new_v.copy_(bits_to_tensor(v, dtype, "cuda"))
        q_t.copy_(bits_to_tensor(q, dtype, "cuda"))
        slots_t.copy_(torch.tensor(sl, dtype=torch.int64))
        ctx_t.copy_(torch.tensor([len(h) for h in hist_k], dtype=torch.int32))
        return q

    def step():
        pkv.reshape_and_cache(new_k, new_v, k_cache, v_cache, slots_t, d_status=st)
        pkv.paged_attention_decode(out_t, q_t, k_cache, v_cache, tables_t, ctx_t, cap, scale, partition_size=P,
                                   workspace=ws, d_status=st)

    def check(q, where):
        ref = np.zeros((S, Hq, D))
        qd = O.decode_bits(q, dtype)
        for s in range(S):
            K = O.decode_bits(np.stack(hist_k[s]), dtype)  # [L, Hkv, D]
            V = O.decode_bits(np.stack(hist_v[s]), dtype)
            for h in range(Hq):
                g = O.kv_head_of(h, Hq, Hkv)
                ref[s, h] = O.attend(qd[s, h][None], K[:, g], V[:, g], scale)[0]
        compare(bits(out_t), ref, dtype, where)

    # one eager step first: the library's one-time host set-up happens outside the capture
    q = stage()
    step()
    torch.cuda.synchronize()
    check(q, "graph case, eager step")

    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for t in range(steps):
        q = stage()
        graph.replay()
        torch.cuda.synchronize()
        check(q, f"graph case, replay {t + 1}")
    assert int(st.item()) == 0
    assert max(len(h) for h in hist_k) <= cap
    del graph


def test_prefill_replayed_from_a_cuda_graph():
    """The chunked prefill of a mixed batch (cache write of the chunks, then
    prefill with its item counter zeroed by a memset node) captured once and
    replayed twice: each replay's output equals the eagerly issued call's bit
    for bit (every work item is computed whole by one CTA, whatever order
    the CTAs take the items in)."""
    from workloads.device import upload_prefill
    b = W.prefill_mixed()
    db = upload_prefill(b)
    st = status_tensor()
    ws = torch.empty(pkv.PREFILL_WORKSPACE_BYTES, dtype=torch.uint8, device="cuda")

    def step(out):
        pkv.reshape_and_cache(db.key, db.value, db.k_cache, db.v_cache, db.slot_mapping, d_status=st)
        pkv.paged_prefill(out, db.q, db.k_cache, db.v_cache, db.block_tables, db.query_start, db.context_lens,
                          b.max_query_len, b.scale, d_status=st, workspace=ws)

    eager = torch.full_like(db.q, float("nan"))
    step(eager)
    torch.cuda.synchronize()
    out = torch.full_like(db.q, float("nan"))
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step(out)
    for _ in range(2):
        out.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), eager.view(torch.int16))
    assert int(st.item()) == 0
    del graph
