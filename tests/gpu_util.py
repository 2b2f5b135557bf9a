"""Helpers shared by the GPU parity tests: device copies of the seeded inputs,
guard-banded output buffers, and the parity metrics with their tolerances.

Tolerances (bf16 inputs, fp32 accumulation, compared with the fp64 oracle on
the very same rounded inputs):
  O    max-abs <= 1e-2 beyond the rounding of O itself to bf16 (half an ulp,
       at most 2^-8 |O_ref|), and relative Frobenius <= 5e-3.  A bf16 output
       cannot be closer than its own rounding: for |O| in [4, 8) half an ulp is
       0.0156, which peaked softmaxes (Q x 8) reach.
  LSE  max-abs <= 1e-3 (natural-log units)
  dQ, dK, dV relative Frobenius <= 1e-2
  FP8  O relative Frobenius <= 3e-2
"""
from __future__ import annotations

import numpy as np
import torch

O_MAX_ABS = 1e-2
O_REL_FRO = 5e-3
LSE_MAX_ABS = 1e-3
GRAD_REL_FRO = 1e-2
FP8_O_REL_FRO = 3e-2
BF16_HALF_ULP_REL = 2.0 ** -8   # bound on half an ulp of bf16, relative to the value

GUARD_BYTES = 4096
SENTINEL = 0xA5


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    """uint16 bf16 bits (host) -> contiguous bf16 CUDA tensor with the same bytes."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.cuda()


def dev_u8(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits)).cuda()


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to(torch.float64).cpu().numpy()


class Guarded:
    """A CUDA buffer with GUARD_BYTES of sentinel bytes on both sides; `view`
    is the tensor handed to the library, `intact()` checks the guards."""

    def __init__(self, shape, dtype):
        elem = torch.empty((), dtype=dtype).element_size()
        n = int(np.prod(shape))
        self.nbytes = n * elem
        self.raw = torch.full((GUARD_BYTES * 2 + self.nbytes,), SENTINEL, dtype=torch.uint8, device="cuda")
        self.view = self.raw[GUARD_BYTES:GUARD_BYTES + self.nbytes].view(dtype).view(shape)

    def intact(self) -> bool:
        head = self.raw[:GUARD_BYTES]
        tail = self.raw[GUARD_BYTES + self.nbytes:]
        return bool(torch.all(head == SENTINEL).item() and torch.all(tail == SENTINEL).item())


def rel_fro(x: np.ndarray, ref: np.ndarray) -> float:
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(x - ref) / (den if den > 0 else 1.0))


def max_abs(x: np.ndarray, ref: np.ndarray) -> float:
    return float(np.max(np.abs(x - ref))) if x.size else 0.0


def assert_o_lse(o, lse, o_ref, lse_ref, what=""):
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse)), f"non-finite output {what}"
    ma, rf, le = max_abs(o, o_ref), rel_fro(o, o_ref), max_abs(lse, lse_ref)
    excess = float(np.max(np.abs(o - o_ref) - BF16_HALF_ULP_REL * np.abs(o_ref))) if o.size else 0.0
    assert excess <= O_MAX_ABS, f"O max-abs beyond bf16 rounding {excess:.3e} > {O_MAX_ABS} (raw {ma:.3e}) {what}"
    assert rf <= O_REL_FRO, f"O rel-Frobenius {rf:.3e} > {O_REL_FRO} {what}"
    assert le <= LSE_MAX_ABS, f"LSE max-abs {le:.3e} > {LSE_MAX_ABS} {what}"
    return ma, rf, le


def sample_rows(N: int, count: int, seed: int) -> np.ndarray:
    """Edge rows (first/last of the sequence and of 128-row tiles) plus seeded random rows."""
    fixed = {0, 1, 127, 128, 129, 255, 256, N // 2, N - 129, N - 128, N - 1}
    rng = np.random.default_rng(seed)
    rnd = rng.integers(0, N, size=count)
    return np.array(sorted(r for r in fixed.union(int(x) for x in rnd) if 0 <= r < N))
