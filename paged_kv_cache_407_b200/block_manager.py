"""Python handle on the C++ block manager (``include/pkv_block_manager.h``).

Argument marshalling only; the free pool, reference counts, Block Tables,
the append rule and copy-on-write live in ``csrc/block_manager.cpp``.  The
arrays it returns are the host-side inputs of one decode step: new-token
slots for ``reshape_and_cache``, block copies for ``copy_blocks`` (run them
first), Block Table rows and context lengths for ``paged_attention_decode``.
"""

from __future__ import annotations

import ctypes

import numpy as np

from .binding import ERR_NO_BLOCKS, PkvError, library


class OutOfBlocks(PkvError):
    """The free pool cannot supply the blocks a call needs; nothing changed."""


def _check(status: int, where: str) -> None:
    if status == ERR_NO_BLOCKS:
        raise OutOfBlocks(status, where)
    if status != 0:
        raise PkvError(status, where)


def _ids(seq_ids) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(seq_ids, dtype=np.int64).reshape(-1))


def _p(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data) if a.size else None


class BlockManager:
    """Free pool of ``num_blocks`` blocks of ``block_size`` tokens and one
    Block Table (at most ``max_blocks_per_seq`` entries) per request."""

    def __init__(self, num_blocks: int, block_size: int, max_blocks_per_seq: int):
        self._lib = library()
        h = ctypes.c_void_p()
        _check(self._lib.pkv_bm_create(num_blocks, block_size, max_blocks_per_seq, ctypes.byref(h)),
               "pkv_bm_create")
        self._h = h
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.max_blocks_per_seq = max_blocks_per_seq

    def close(self) -> None:
        if getattr(self, "_h", None):
            self._lib.pkv_bm_destroy(self._h)
            self._h = None

    def __del__(self):
        self.close()

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    # -- queries ------------------------------------------------------------
    @property
    def num_free_blocks(self) -> int:
        return self._lib.pkv_bm_num_free_blocks(self._h)

    @property
    def num_sequences(self) -> int:
        return self._lib.pkv_bm_num_sequences(self._h)

    def ref_count(self, block: int) -> int:
        return self._lib.pkv_bm_ref_count(self._h, block)

    def context_len(self, seq_id: int) -> int:
        return self._lib.pkv_bm_context_len(self._h, seq_id)

    def free_list(self) -> np.ndarray:
        n = ctypes.c_int32()
        out = np.empty(self.num_blocks, np.int32)
        _check(self._lib.pkv_bm_free_list(self._h, _p(out), out.size, ctypes.byref(n)), "pkv_bm_free_list")
        return out[: n.value].copy()

    def blocks_needed(self, seq_ids) -> int:
        ids = _ids(seq_ids)
        n = self._lib.pkv_bm_blocks_needed(self._h, _p(ids), ids.size)
        if n < 0:
            raise PkvError(11, "pkv_bm_blocks_needed")
        return n

    # -- requests -----------------------------------------------------------
    def add_sequence(self, seq_id: int, num_tokens: int) -> np.ndarray:
        """A new request of ``num_tokens`` prompt tokens; returns their slots."""
        slots = np.empty(num_tokens, np.int64)
        _check(self._lib.pkv_bm_add_sequence(self._h, seq_id, num_tokens, _p(slots)), "pkv_bm_add_sequence")
        return slots

    def fork(self, parent_id: int, child_id: int) -> None:
        _check(self._lib.pkv_bm_fork(self._h, parent_id, child_id), "pkv_bm_fork")

    def free_sequence(self, seq_id: int) -> None:
        _check(self._lib.pkv_bm_free_sequence(self._h, seq_id), "pkv_bm_free_sequence")

    def append(self, seq_ids) -> tuple[np.ndarray, np.ndarray]:
        """One decode step: one new token per listed request.  Returns the
        slots ``int64 [n]`` and the block copies ``int64 [k, 2]`` (src, dst)."""
        ids = _ids(seq_ids)
        slots = np.empty(ids.size, np.int64)
        pairs = np.empty((max(ids.size, 1), 2), np.int64)
        k = ctypes.c_int32()
        _check(self._lib.pkv_bm_append(self._h, _p(ids), ids.size, _p(slots), _p(pairs), ids.size,
                                       ctypes.byref(k)), "pkv_bm_append")
        return slots, pairs[: k.value].copy()

    def block_tables(self, seq_ids, row_stride: int | None = None) -> tuple[np.ndarray, np.ndarray]:
        """Block Table rows ``int32 [n, row_stride]`` padded with -1 and the
        context lengths ``int32 [n]`` of the listed requests."""
        ids = _ids(seq_ids)
        stride = self.max_blocks_per_seq if row_stride is None else row_stride
        tables = np.empty((ids.size, stride), np.int32)
        lens = np.empty(ids.size, np.int32)
        _check(self._lib.pkv_bm_block_tables(self._h, _p(ids), ids.size, _p(tables), stride, _p(lens)),
               "pkv_bm_block_tables")
        return tables, lens
