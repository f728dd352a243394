"""Move a ``PagedBatch`` to the GPU as torch tensors (and bits back).

Plumbing only: device memory comes from torch, every value comes from the
seeded generator in ``workloads``.
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

from . import BF16, F16, PagedBatch

TORCH_DTYPE = {F16: torch.float16, BF16: torch.bfloat16}


def bits_to_tensor(bits: np.ndarray, dtype: str, device) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.to(device).view(TORCH_DTYPE[dtype])


def tensor_to_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


@dataclass
class DeviceBatch:
    q: torch.Tensor
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    block_tables: torch.Tensor
    context_lens: torch.Tensor
    key: torch.Tensor
    value: torch.Tensor
    slot_mapping: torch.Tensor
    cow_pairs: torch.Tensor
    block_tables_before_cow: torch.Tensor | None
    out: torch.Tensor


def upload(b: PagedBatch, device="cuda") -> DeviceBatch:
    q = bits_to_tensor(b.q, b.dtype, device)
    return DeviceBatch(
        q=q,
        k_cache=bits_to_tensor(b.k_cache, b.dtype, device),
        v_cache=bits_to_tensor(b.v_cache, b.dtype, device),
        block_tables=torch.from_numpy(b.block_tables).to(device),
        context_lens=torch.from_numpy(b.context_lens).to(device),
        key=bits_to_tensor(b.key, b.dtype, device),
        value=bits_to_tensor(b.value, b.dtype, device),
        slot_mapping=torch.from_numpy(b.slot_mapping).to(device),
        cow_pairs=torch.from_numpy(np.ascontiguousarray(b.cow_pairs)).to(device),
        block_tables_before_cow=(None if b.block_tables_before_cow is None
                                 else torch.from_numpy(b.block_tables_before_cow).to(device)),
        out=torch.empty_like(q),
    )


@dataclass
class DeviceFp8Batch:
    q: torch.Tensor
    k_cache: torch.Tensor  # uint8 [N, Hkv, B, D]
    v_cache: torch.Tensor  # uint8 [N, Hkv, D, B]
    block_tables: torch.Tensor
    context_lens: torch.Tensor
    key: torch.Tensor
    value: torch.Tensor
    slot_mapping: torch.Tensor
    cow_pairs: torch.Tensor
    out: torch.Tensor


def upload_fp8(f8, device="cuda") -> DeviceFp8Batch:
    b = f8.base
    q = bits_to_tensor(b.q, b.dtype, device)
    return DeviceFp8Batch(
        q=q,
        k_cache=torch.from_numpy(f8.k_cache).to(device),
        v_cache=torch.from_numpy(f8.v_cache).to(device),
        block_tables=torch.from_numpy(b.block_tables).to(device),
        context_lens=torch.from_numpy(b.context_lens).to(device),
        key=bits_to_tensor(b.key, b.dtype, device),
        value=bits_to_tensor(b.value, b.dtype, device),
        slot_mapping=torch.from_numpy(b.slot_mapping).to(device),
        cow_pairs=torch.from_numpy(np.ascontiguousarray(b.cow_pairs)).to(device),
        out=torch.empty_like(q),
    )


@dataclass
class DevicePrefillBatch:
    q: torch.Tensor
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    block_tables: torch.Tensor
    context_lens: torch.Tensor
    query_start: torch.Tensor
    key: torch.Tensor
    value: torch.Tensor
    slot_mapping: torch.Tensor
    out: torch.Tensor


def upload_prefill(b, device="cuda") -> DevicePrefillBatch:
    q = bits_to_tensor(b.q, b.dtype, device)
    return DevicePrefillBatch(
        q=q,
        k_cache=bits_to_tensor(b.k_cache, b.dtype, device),
        v_cache=bits_to_tensor(b.v_cache, b.dtype, device),
        block_tables=torch.from_numpy(b.block_tables).to(device),
        context_lens=torch.from_numpy(b.context_lens).to(device),
        query_start=torch.from_numpy(b.query_start).to(device),
        key=bits_to_tensor(b.key, b.dtype, device),
        value=bits_to_tensor(b.value, b.dtype, device),
        slot_mapping=torch.from_numpy(b.slot_mapping).to(device),
        out=torch.empty_like(q),
    )
