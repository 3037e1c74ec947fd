"""Move a Workload's host arrays into device tensors (marshalling only)."""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch


def bf16_tensor(bits: np.ndarray, device="cuda") -> torch.Tensor:
    """uint16 bf16 bit patterns -> torch.bfloat16 tensor (no rounding)."""
    t = torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(
        np.int16))
    return t.view(torch.bfloat16).to(device)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """torch.bfloat16 tensor -> uint16 bit patterns on the host."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(
        np.uint16)


def i32_tensor(a: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)


@dataclass
class DeviceBatch:
    q: torch.Tensor
    k_pool: torch.Tensor
    v_pool: torch.Tensor
    block_tables: torch.Tensor
    context_lens: torch.Tensor
    k_new: torch.Tensor
    v_new: torch.Tensor
    slot_mapping: torch.Tensor
    query_start_loc: torch.Tensor
    err: torch.Tensor


def upload(wl, device="cuda") -> DeviceBatch:
    return DeviceBatch(
        q=bf16_tensor(wl.q, device),
        k_pool=bf16_tensor(wl.k_pool, device),
        v_pool=bf16_tensor(wl.v_pool, device),
        block_tables=i32_tensor(wl.block_tables, device),
        context_lens=i32_tensor(wl.context_lens, device),
        k_new=bf16_tensor(wl.k_new, device),
        v_new=bf16_tensor(wl.v_new, device),
        slot_mapping=i32_tensor(wl.slot_mapping, device),
        query_start_loc=i32_tensor(wl.query_start_loc, device),
        err=torch.zeros(1, dtype=torch.int32, device=device),
    )
