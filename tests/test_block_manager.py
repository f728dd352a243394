"""The C++ block manager (libpkv, host only) against the oracle block
manager, decision for decision: slots, copy pairs, Block Tables, lengths,
reference counts and the order of the free pool (CPU only)."""

import numpy as np
import pytest

import oracle.block_manager as BMO
from paged_kv_cache_407_b200 import PkvError
from paged_kv_cache_407_b200.block_manager import BlockManager, OutOfBlocks


@pytest.fixture(scope="module", autouse=True)
def _built():
    from paged_kv_cache_407_b200.build import build
    build()


def _same_state(cm, om, ids=None):
    assert cm.free_list().tolist() == list(om.free)
    assert [cm.ref_count(b) for b in range(om.num_blocks)] == om.ref
    assert cm.num_sequences == len(om.tables)
    ids = sorted(om.tables) if ids is None else ids
    if ids:
        tables, lens = cm.block_tables(ids)
        rows, olens = om.block_tables(ids)
        assert tables.tolist() == rows and lens.tolist() == olens


@pytest.mark.parametrize("seed", range(8))
def test_churn_matches_oracle(seed):
    rng = np.random.default_rng(100 + seed)
    B = int(rng.choice([1, 2, 8, 16, 32]))
    N = int(rng.integers(4, 60))
    M = int(rng.integers(2, 12))
    cm = BlockManager(N, B, M)
    om = BMO.BlockManager(N, B, M)
    next_id = 1000
    for _ in range(300):
        live = sorted(om.tables)
        op = rng.random()
        if op < 0.2 or not live:
            n = int(rng.integers(0, B * M + 2))
            try:
                exp = om.add_sequence(next_id, n)
            except (BMO.OutOfBlocks, ValueError) as e:
                with pytest.raises(OutOfBlocks if isinstance(e, BMO.OutOfBlocks) else PkvError):
                    cm.add_sequence(next_id, n)
            else:
                assert cm.add_sequence(next_id, n).tolist() == exp
            next_id += 1
        elif op < 0.3:
            p = int(rng.choice(live))
            om.fork(p, next_id)
            cm.fork(p, next_id)
            next_id += 1
        elif op < 0.42:
            s = int(rng.choice(live))
            om.free_sequence(s)
            cm.free_sequence(s)
        else:
            ids = [int(x) for x in rng.permutation(live)[: int(rng.integers(1, len(live) + 1))]]
            assert cm.blocks_needed(ids) == om.blocks_needed(ids)
            try:
                exp_slots, exp_copies = om.append(ids)
            except (BMO.OutOfBlocks, ValueError) as e:
                with pytest.raises(OutOfBlocks if isinstance(e, BMO.OutOfBlocks) else PkvError):
                    cm.append(ids)
            else:
                slots, copies = cm.append(ids)
                assert slots.tolist() == exp_slots
                assert [tuple(c) for c in copies.tolist()] == exp_copies
        _same_state(cm, om)
    cm.close()


def test_copy_on_write_of_a_forked_prefix():
    """A 1016-token prefix (last block half full) forked to 8 requests: the
    first decode step copies the shared last block for all but the last
    request, which writes into it in place."""
    B = 16
    cm = BlockManager(200, B, 80)
    cm.add_sequence(0, 1016)
    for c in range(1, 9):
        cm.fork(0, c)
    cm.free_sequence(0)
    assert cm.ref_count(0) == 8 and cm.ref_count(63) == 8
    slots, copies = cm.append(list(range(1, 9)))
    assert copies.shape == (7, 2) and (copies[:, 0] == 63).all()
    assert len(set(copies[:, 1].tolist())) == 7
    assert slots[-1] == 63 * B + 1016 % B
    tables, lens = cm.block_tables(list(range(1, 9)))
    assert (lens == 1017).all() and (tables[:, :63] == np.arange(63)).all()
    assert cm.ref_count(63) == 1


def test_errors_change_nothing():
    cm = BlockManager(4, 4, 3)
    cm.add_sequence(1, 8)  # blocks 0, 1
    cm.add_sequence(2, 4)  # block 2
    before = (cm.free_list().tolist(), cm.block_tables([1, 2]))
    with pytest.raises(PkvError):
        cm.add_sequence(1, 3)  # id present
    with pytest.raises(PkvError):
        cm.fork(7, 8)  # unknown parent
    with pytest.raises(PkvError):
        cm.append([1, 1])  # repeated id
    with pytest.raises(PkvError):
        cm.append([3])  # unknown id
    with pytest.raises(OutOfBlocks):
        cm.add_sequence(3, 5)  # needs 2 blocks, 1 free
    cm.append([1])  # takes block 3
    with pytest.raises(OutOfBlocks):
        cm.append([2])  # block 2 full, pool empty
    with pytest.raises(PkvError):
        BlockManager(4, 4, 2).add_sequence(0, 9)  # 3 blocks > table of 2
    assert cm.free_list().tolist() == [] and cm.context_len(1) == 9
    tables, lens = cm.block_tables([1, 2])
    assert tables.tolist() == [[0, 1, 3], [2, -1, -1]] and lens.tolist() == [9, 4]
    assert before[0] == [3]
    cm.free_sequence(1)
    cm.free_sequence(2)
    assert cm.free_list().tolist() == [0, 1, 3, 2]
    assert cm.context_len(1) == -1 and cm.ref_count(9) == -1


def test_host_arrays_feed_the_device_calls():
    """Shapes and dtypes of one step's arrays are the decode inputs."""
    cm = BlockManager(64, 16, 8)
    for s in range(5):
        cm.add_sequence(s, 10 + 7 * s)
    slots, copies = cm.append(range(5))
    tables, lens = cm.block_tables(range(5), row_stride=10)
    assert slots.dtype == np.int64 and slots.shape == (5,)
    assert copies.dtype == np.int64 and copies.shape == (0, 2)
    assert tables.dtype == np.int32 and tables.shape == (5, 10) and (tables[:, 8:] == -1).all()
    assert lens.dtype == np.int32 and lens.tolist() == [11 + 7 * s for s in range(5)]



def test_concurrent_native_threads_keep_one_manager_consistent(tmp_path):
    """Calls on one manager are serialised by its lock.  tests/native/
    bm_threads.cpp, built against libpkv.so, runs eight host threads that
    add, fork, extend and free their own requests on one shared pool (which
    runs dry, so steps are refused too) and then checks the lengths, the
    reference counts and the free pool against what the threads did.  Built
    from the same source with the lock taken out, that program crashes or
    reports inconsistencies."""
    import os
    import shutil
    import subprocess
    from paged_kv_cache_407_b200.build import INCLUDE, LIB_PATH
    cxx = os.environ.get("CXX") or shutil.which("g++") or shutil.which("c++")
    assert cxx, "a host C++ compiler is needed"
    src = os.path.join(os.path.dirname(os.path.abspath(__file__)), "native", "bm_threads.cpp")
    exe = str(tmp_path / "bm_threads")
    libdir = os.path.dirname(LIB_PATH)
    subprocess.run([cxx, "-O2", "-std=c++17", "-pthread", "-I", INCLUDE, src, "-L", libdir, "-lpkv",
                    f"-Wl,-rpath,{libdir}", "-o", exe], check=True, capture_output=True, text=True)
    for threads, steps in ((8, 4000), (16, 2000)):
        res = subprocess.run([exe, str(threads), str(steps)], capture_output=True, text=True, timeout=120)
        assert res.returncode == 0 and "inconsistencies 0" in res.stdout, (res.returncode, res.stdout, res.stderr)
