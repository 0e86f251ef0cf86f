"""Device residency of quantised weights (plumbing: torch allocations only).

A q-matrix arrives as host arrays (q uint32 words, s/b bf16 bits) and is
copied to the device unchanged.  A routed layer's E expert blobs live in one
device allocation with a fixed stride; `blob_ptrs` is the device table of
their addresses that the kernels read.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional

import numpy as np
import torch

from ._lib import moe_qmat, qmat


@dataclass
class DeviceQMat:
    q: torch.Tensor
    s: torch.Tensor
    b: torch.Tensor
    out: int
    inn: int
    bits: int

    @property
    def c(self) -> moe_qmat:
        return qmat(self.q, self.s, self.b, self.out, self.inn, self.bits)


def _dev(a: np.ndarray, dtype, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(dtype)).to(device)


def upload_qmat(m, device="cuda") -> DeviceQMat:
    return DeviceQMat(_dev(m.q, np.int32, device), _dev(m.s, np.int16, device), _dev(m.b, np.int16, device),
                      m.out, m.inn, m.bits)


def blob_table(blobs: torch.Tensor) -> torch.Tensor:
    """Device int64 [E] of the addresses of the rows of a [E, stride] uint8 tensor."""
    E, stride = blobs.shape
    base = blobs.data_ptr()
    return torch.tensor([base + e * stride for e in range(E)], dtype=torch.int64, device=blobs.device)


@dataclass
class DeviceLayer:
    router: DeviceQMat
    bias: Optional[torch.Tensor]
    shared: List[DeviceQMat]
    blobs: torch.Tensor          # uint8 [E, stride] (device)
    blob_ptrs: torch.Tensor      # int64 [E] (device)

    @property
    def shared_c(self):
        return [m.c for m in self.shared]


def upload_layer(router, bias, shared, blobs_host: np.ndarray, device="cuda") -> DeviceLayer:
    blobs = torch.from_numpy(blobs_host).to(device)
    b = None if bias is None else torch.from_numpy(np.ascontiguousarray(bias, dtype=np.float32)).to(device)
    return DeviceLayer(upload_qmat(router, device), b, [upload_qmat(m, device) for m in shared], blobs,
                       blob_table(blobs))
