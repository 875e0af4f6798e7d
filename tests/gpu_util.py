"""Helpers for the GPU parity tests: device buffers with canary guard bands and
conversions between torch tensors and the oracle's numpy arrays.

Inputs always come from the seeded generators in ``workloads`` or from the
oracle; expected values always come from the oracle (never from the CUDA path).
"""
from __future__ import annotations

import numpy as np
import torch

GUARD = 4096          # bytes of canary on each side of every output buffer
CANARY = 0xA5


class Guarded:
    """A device tensor view with canary-filled guard bands on both sides."""

    def __init__(self, shape, dtype, device="cuda", fill=None):
        nbytes = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.raw = torch.full((nbytes + 2 * GUARD,), CANARY, dtype=torch.uint8, device=device)
        if fill is not None:
            self.raw[GUARD:GUARD + nbytes].fill_(fill)
        self.t = self.raw[GUARD:GUARD + nbytes].view(dtype).view(*shape)
        assert self.t.data_ptr() % 16 == 0

    def guards_intact(self) -> bool:
        head = self.raw[:GUARD]
        tail = self.raw[self.raw.numel() - GUARD:]
        return bool((head == CANARY).all().item() and (tail == CANARY).all().item())


def to_dev_codes(q: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(q)).cuda()


def to_dev_f32(s: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(s, dtype=np.float32)).cuda()


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def tolerance_report(y: np.ndarray, ref: np.ndarray):
    """(all within |y-ref| <= 1e-2 |ref| + 2e-3 rms(ref), worst excess ratio, rms)."""
    ref = np.asarray(ref, dtype=np.float64)
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    bound = 1e-2 * np.abs(ref) + 2e-3 * rms
    err = np.abs(np.asarray(y, dtype=np.float64) - ref)
    ratio = float((err / np.maximum(bound, 1e-300)).max()) if ref.size else 0.0
    return bool(np.all(err <= bound)), ratio, rms
