"""Seeded cases copied to a CUDA device as torch tensors.

Input plumbing only: the host arrays of a PagedDecodeCase / PagedPrefillCase
are copied bit for bit (bf16 and fp16 values travel as their 16-bit
patterns).  Nothing here computes any part of the attention, and nothing here
imports the library or the oracle; the benchmark, the smoke check and the GPU
tests all upload through these functions.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

from .workloads import DTYPE_BF16, DTYPE_F16, DTYPE_F32

# pa_dtype codes of the C ABI (include/pagedattn.h)
DTYPE_CODE = {DTYPE_F32: 0, DTYPE_BF16: 1, DTYPE_F16: 2}


def to_device(a: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    """A value array of a case as a torch tensor of its own dtype."""
    a = np.ascontiguousarray(a)
    if dtype == DTYPE_BF16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
    if dtype == DTYPE_F16:
        return torch.from_numpy(a.view(np.int16)).view(torch.float16).to(device)
    return torch.from_numpy(a).to(device)


def ints_to_device(a: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)


@dataclass
class DeviceCase:
    q: torch.Tensor
    k_new: torch.Tensor
    v_new: torch.Tensor
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    block_tables: torch.Tensor
    context_lens: torch.Tensor
    slot_mapping: torch.Tensor
    out: torch.Tensor


def upload(case, device="cuda") -> DeviceCase:
    """A decode case on the device; `out` is filled with NaN."""
    v = lambda a: to_device(a, case.dtype, device)
    q = v(case.q)
    return DeviceCase(q=q, k_new=v(case.k_new), v_new=v(case.v_new), k_cache=v(case.k_cache),
                      v_cache=v(case.v_cache), block_tables=ints_to_device(case.block_tables, device),
                      context_lens=ints_to_device(case.context_lens, device),
                      slot_mapping=ints_to_device(case.slot_mapping, device), out=torch.full_like(q, float("nan")))


def upload_prefill(pc, device="cuda") -> dict:
    """A prefill case on the device (a dict of tensors); `out` is filled with NaN."""
    v = lambda a: to_device(a, pc.dtype, device)
    i = lambda a: ints_to_device(a, device)
    q = v(pc.q)
    return dict(q=q, k_new=v(pc.k_new), v_new=v(pc.v_new), k_cache=v(pc.k_cache), v_cache=v(pc.v_cache),
                block_tables=i(pc.block_tables), context_lens=i(pc.context_lens), query_start=i(pc.query_start),
                slot_mapping=i(pc.slot_mapping), out=torch.full_like(q, float("nan")))


def shape_fields(case, B: int | None = None) -> tuple:
    """The eight pa_shape fields of a case, in declaration order (B may be
    overridden: a prefill append writes one row per new token)."""
    return (case.B if B is None else B, case.Hq, case.Hkv, case.D, case.block_size, case.num_blocks,
            case.max_blocks_per_seq, DTYPE_CODE[case.dtype])
