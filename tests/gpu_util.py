"""Helpers for the GPU parity tests: host <-> device in the oracle's storage
conventions (bf16/fp16 as uint16 bits) and guard-banded device buffers that
detect writes outside a collective's output."""
from __future__ import annotations

import numpy as np
import pytest
import torch

TORCH = {"bf16": torch.bfloat16, "fp16": torch.float16, "fp32": torch.float32, "int32": torch.int32}
VIEW = {"bf16": torch.int16, "fp16": torch.int16, "fp32": torch.float32, "int32": torch.int32}
NPV = {"bf16": np.int16, "fp16": np.int16, "fp32": np.float32, "int32": np.int32}
NPS = {"bf16": np.uint16, "fp16": np.uint16, "fp32": np.float32, "int32": np.int32}
ESIZE = {"bf16": 2, "fp16": 2, "fp32": 4, "int32": 4}
GUARD = 4096  # bytes of canary on each side
CANARY = 0xA5


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def to_dev(a: np.ndarray, dtype: str) -> torch.Tensor:
    a = np.ascontiguousarray(a, dtype=NPS[dtype]).view(NPV[dtype])
    return torch.from_numpy(a.copy()).view(TORCH[dtype]).cuda()


def from_dev(t: torch.Tensor, dtype: str) -> np.ndarray:
    return t.detach().contiguous().view(VIEW[dtype]).cpu().numpy().view(NPS[dtype])


class Guarded:
    """A device buffer of ``count`` elements with canary bands around it.

    ``offset`` shifts the data by that many bytes from a 256-byte boundary,
    to exercise the unaligned paths."""

    def __init__(self, count: int, dtype: str, offset: int = 0, fill: np.ndarray | None = None):
        self.dtype = dtype
        self.count = count
        es = ESIZE[dtype]
        self.nbytes = count * es
        self.offset = offset
        total = GUARD + offset + self.nbytes + GUARD
        self.raw = torch.full((total,), CANARY, dtype=torch.uint8, device="cuda")
        lo = GUARD + offset
        self.bytes_view = self.raw[lo:lo + self.nbytes]
        if fill is not None:
            src = np.ascontiguousarray(fill, dtype=NPS[dtype]).view(np.uint8)
            self.bytes_view.copy_(torch.from_numpy(src.copy()).cuda())
        # a typed view needs element alignment; uint8 storage offset keeps the pointer exact
        self.t = self.bytes_view.view(TORCH[dtype]) if (lo % es == 0) else None

    @property
    def ptr(self) -> int:
        return self.bytes_view.data_ptr()

    def host(self) -> np.ndarray:
        return self.bytes_view.cpu().numpy().view(NPS[self.dtype]).copy()

    def guards_intact(self) -> bool:
        lo = GUARD + self.offset
        g = torch.cat([self.raw[:lo], self.raw[lo + self.nbytes:]])
        return bool((g == CANARY).all().item())


def status_tensor() -> torch.Tensor:
    return torch.zeros(2, dtype=torch.int32, device="cuda")
