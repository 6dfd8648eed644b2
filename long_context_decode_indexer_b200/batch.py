"""Device-side plumbing: put a host batch (synth.Inputs) into torch-owned device
memory and build the C-ABI structs that describe it.  No arithmetic of the
method happens here; torch only owns the memory."""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch

from . import dsa
from .synth import Inputs


@dataclasses.dataclass
class DeviceBatch:
    inp: Inputs
    q_idx: torch.Tensor
    w: torch.Tensor
    kidx: torch.Tensor
    k_scale: Optional[torch.Tensor]
    q: torch.Tensor
    kv: torch.Tensor
    q_seq: torch.Tensor
    q_n: torch.Tensor
    seq_row0: Optional[torch.Tensor]
    page_table: Optional[torch.Tensor]

    def params(self, *, topk=None, max_n=None, q_per_seq=None) -> dsa.Params:
        i = self.inp
        return dsa.make_params(nq=i.nq, h_idx=i.h_idx, d_idx=i.d_idx, h=i.h,
                               topk=i.topk if topk is None else topk,
                               max_n=i.max_n if max_n is None else max_n,
                               q_per_seq=i.q_per_seq if q_per_seq is None else q_per_seq,
                               scale=i.scale)

    def kvdesc(self) -> dsa.KV:
        return dsa.make_kv(q_seq=self.q_seq, q_n=self.q_n, seq_row0=self.seq_row0,
                           page_table=self.page_table, page_size=self.inp.page_size,
                           cache_rows=self.kidx.shape[0])

    @property
    def kv_row_stride(self) -> int:
        return int(self.kv.stride(0))


def _dev(a: np.ndarray, device, dtype=None) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.to(device, non_blocking=False)


def upload(inp: Inputs, device="cuda") -> DeviceBatch:
    return DeviceBatch(
        inp=inp,
        q_idx=_dev(inp.q_idx, device),
        w=_dev(inp.w.view(np.int16), device),
        kidx=_dev(inp.kidx, device),
        k_scale=None if inp.k_scale is None else _dev(inp.k_scale, device),
        q=_dev(inp.q.view(np.int16), device),
        kv=_dev(inp.kv.view(np.int16), device),
        q_seq=_dev(inp.q_seq, device),
        q_n=_dev(inp.q_n, device),
        seq_row0=None if inp.seq_row0 is None else _dev(inp.seq_row0, device),
        page_table=None if inp.page_table is None else _dev(inp.page_table, device),
    )


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A zero-filled, 256-byte aligned device buffer of at least nbytes (the
    C ABI wants the workspace zeroed before its first use; torch's caching
    allocator returns 512-byte aligned blocks)."""
    t = torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device)
    assert t.data_ptr() % 256 == 0
    return t


def bf16_bits_to_float(t: torch.Tensor) -> torch.Tensor:
    """Reinterpret int16 storage of bf16 values as float32 (no rounding)."""
    return t.view(torch.bfloat16).float()
