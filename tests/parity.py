"""Helpers shared by the GPU parity tests: run a batch through the C-ABI
binding and compare with the oracle.

Tolerance for attention outputs (fp16/bf16 storage, fp32 accumulation): a
maximum absolute error of 2e-3 and a maximum relative error of 1e-2.

* Every output, fp16 or bf16, must satisfy the combined per-element bound
  |gpu - oracle| <= ATOL + RTOL * |oracle| (ATOL = 2e-3, RTOL = 1e-2).
* fp16 outputs must also satisfy the two limits literally and separately:
  max |gpu - oracle| <= 2e-3 over every element, and max |gpu - oracle| /
  |oracle| <= 1e-2 over the elements with |oracle| >= 0.2 (below that the
  relative error of a value near zero says nothing).
* bf16 outputs are held to the combined bound only: rounding the exact result
  to bf16 alone moves a value in [1, 2) by up to 2^-8 (3.9e-3), so a plain
  absolute bound of 2e-3 cannot hold for every element of a bf16 output.
  The statistics record that storage floor beside the measured error.

Cache writes and block copies must match bit for bit.  Every comparison's
statistics are kept in RECORDS and printed at the end of the pytest run.
"""

from __future__ import annotations

import numpy as np
import torch

import oracle as O
import paged_kv_cache_407_b200 as pkv
from workloads.device import tensor_to_bits, upload

ATOL = 2e-3
RTOL = 1e-2


LITERAL_REL_FLOOR = 0.2  # relative errors are taken over |oracle| >= this

# (where, dtype, statistics) of every comparison made in this process
RECORDS: list[tuple[str, str, dict]] = []


def error_stats(got: np.ndarray, ref: np.ndarray, dtype: str) -> dict:
    """Maximum absolute and relative errors of float64 values ``got`` against
    ``ref``, the error that rounding ``ref`` to ``dtype`` alone would leave,
    and whether the combined and the literal bounds hold."""
    err = np.abs(got - ref)
    big = np.abs(ref) >= LITERAL_REL_FLOOR
    floor = np.abs(O.decode_bits(O.encode_bits(ref, dtype), dtype) - ref)
    max_abs = float(err.max())
    max_rel = float((err[big] / np.abs(ref[big])).max()) if big.any() else 0.0
    return {
        "max_abs": max_abs,
        "max_rel": max_rel,
        "storage_floor_abs": float(floor.max()),
        "combined_ok": bool(np.all(err <= ATOL + RTOL * np.abs(ref))),
        "literal_ok": bool(max_abs <= ATOL and max_rel <= RTOL),
        "n": int(err.size),
    }


def compare(gpu_bits: np.ndarray, ref: np.ndarray, dtype: str, where: str = "",
            literal: bool | None = None) -> dict:
    """Element-wise check of fp16/bf16 GPU output bits against float64 oracle
    values (rows of ``ref`` that are NaN are not compared).  Asserts the
    combined bound always and the literal limits when ``literal`` (default:
    for fp16 outputs); returns the statistics."""
    got = O.decode_bits(gpu_bits, dtype)
    rows = ~np.isnan(ref).any(axis=-1)
    got, ref = got[rows], ref[rows]
    assert got.size > 0, "nothing compared"
    if literal is None:
        literal = dtype == "f16"
    stats = error_stats(got, ref, dtype)
    RECORDS.append((where, dtype, stats))
    err = np.abs(got - ref)
    bad = ~(err <= ATOL + RTOL * np.abs(ref))
    if bad.any():
        idx = np.argwhere(bad)[0]
        raise AssertionError(
            f"{where}: {int(bad.sum())} of {bad.size} elements outside {ATOL} + {RTOL}|ref|; "
            f"first at {tuple(idx)}: gpu={got[tuple(idx)]!r} ref={ref[tuple(idx)]!r}; "
            f"max abs err {err.max():.3e}")
    if literal:
        assert stats["literal_ok"], (
            f"{where}: max abs err {stats['max_abs']:.3e} (limit {ATOL}) / max rel err "
            f"{stats['max_rel']:.3e} over |ref| >= {LITERAL_REL_FLOOR} (limit {RTOL})")
    return stats


def status_tensor(device="cuda"):
    return torch.zeros(1, dtype=torch.int32, device=device)


def run_step(batch, *, device="cuda", partition_size=None, write=True, cow=True, d_status=None,
             tables=None):
    """One decode step through the library: copy-on-write pairs, the cache
    write of the new tokens, then decode attention.  Returns the DeviceBatch."""
    db = upload(batch, device)
    if cow and batch.cow_pairs.shape[0]:
        pkv.copy_blocks(db.k_cache, db.v_cache, db.cow_pairs, d_status=d_status)
    if write and batch.num_tokens:
        pkv.reshape_and_cache(db.key, db.value, db.k_cache, db.v_cache, db.slot_mapping, d_status=d_status)
    P = batch.partition_size if partition_size is None else partition_size
    pkv.paged_attention_decode(db.out, db.q, db.k_cache, db.v_cache,
                               db.block_tables if tables is None else tables, db.context_lens,
                               batch.max_context_len, batch.scale, partition_size=P, d_status=d_status)
    torch.cuda.synchronize()
    return db


def oracle_caches(batch, write=True, cow=True):
    kc, vc = batch.k_cache, batch.v_cache
    if cow and batch.cow_pairs.shape[0]:
        kc, vc = O.copy_blocks(kc, vc, batch.cow_pairs)
    if write and batch.num_tokens:
        kc, vc = O.reshape_and_cache(kc, vc, batch.key, batch.value, batch.slot_mapping, batch.block_size)
    return kc, vc


def oracle_out(batch, kc, vc, seqs=None):
    return O.paged_attention_decode(batch.q, kc, vc, batch.block_tables, batch.context_lens,
                                    batch.block_size, batch.scale, batch.dtype, seqs=seqs)


def bits(t):
    return tensor_to_bits(t)
