"""GPU parity on the five named workloads at full size, in the launch
configuration the benchmark times (B200 only).  The oracle computes a seeded
sample of sequences one by one; cache writes and block copies are compared
over the whole pool."""

import numpy as np
import pytest
import torch

import paged_kv_cache_407_b200 as pkv
import workloads as W
from parity import bits, compare, oracle_caches, oracle_out, run_step, status_tensor

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "these tests need a CUDA device"
    from paged_kv_cache_407_b200.build import build
    build()
    pkv.library()


def _sample(n_seqs, k, seed):
    rng = np.random.default_rng(seed)
    return sorted(rng.choice(n_seqs, size=min(k, n_seqs), replace=False).tolist())


def _check_workload(batch, sample, check_pool=True):
    st = status_tensor()
    db = run_step(batch, d_status=st)
    assert int(st.item()) == 0
    kc, vc = oracle_caches(batch)
    if check_pool:
        assert np.array_equal(bits(db.k_cache), kc), "K pool differs after write/copy"
        assert np.array_equal(bits(db.v_cache), vc), "V pool differs after write/copy"
    ref = oracle_out(batch, kc, vc, seqs=sample)
    return compare(bits(db.out), ref, batch.dtype, batch.name)


# fp16 workloads meet the 2e-3 / 1e-2 limits literally; bf16 ones the
# combined per-element bound (a bf16 output cannot meet 2e-3 absolute in
# [1, 2) after its own rounding).

def test_tiny_every_output():
    b = W.tiny()
    stats = _check_workload(b, None)
    assert stats["n"] == 4 * 4 * 64
    assert stats["literal_ok"], stats


def test_llama7b_mha_sampled():
    b = W.llama7b_mha()
    stats = _check_workload(b, _sample(b.num_seqs, 8, 2))
    assert stats["literal_ok"], stats


def test_gqa_write_sampled():
    b = W.gqa_write()
    stats = _check_workload(b, _sample(b.num_seqs, 24, 3))
    assert stats["combined_ok"], stats


def test_prefix_share_sampled():
    b = W.prefix_share()
    stats = _check_workload(b, _sample(b.num_seqs, 12, 4))
    assert stats["literal_ok"], stats


def test_long_context_sampled():
    b = W.long_context()
    assert b.partition_size == 512
    stats = _check_workload(b, [1, 3], check_pool=False)
    assert stats["combined_ok"], stats
