"""Helpers for the GPU parity tests: tolerances, canaries, input transfer."""
from __future__ import annotations

import numpy as np
import torch

# Tolerance for bf16 outputs against the fp64 oracle: |err| <= 1e-2 + 1.6e-2 |ref|.
BF16_ATOL = 1e-2
BF16_RTOL = 1.6e-2
# fp32 cos/sin planes: |err| <= 2e-6 |ref|.
PLANE_RTOL = 2e-6
# Normalised-MSE bar (vllm.cpp #185 gates its reducing kernels at 5e-4).
NMSE_BAR = 5e-4

SENTINEL_BF16 = 0x7FB7   # a NaN pattern no kernel writes
SENTINEL_F32 = 0x7FC0DEAD


def to_dev(t: torch.Tensor) -> torch.Tensor:
    return t.to("cuda")


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_bf16_close(got: torch.Tensor, ref: np.ndarray, what: str = "") -> dict:
    g = bf16_to_f64(got).reshape(ref.shape)
    err = np.abs(g - ref)
    bound = BF16_ATOL + BF16_RTOL * np.abs(ref)
    bad = ~(err <= bound)
    if bad.any():
        idx = np.argwhere(bad)[:5]
        rows = ["%s: got %r ref %r" % (tuple(i), g[tuple(i)], ref[tuple(i)]) for i in idx]
        raise AssertionError("%s: %d of %d outside |err| <= 1e-2 + 1.6e-2|ref|; first: %s"
                             % (what, int(bad.sum()), bad.size, "; ".join(rows)))
    denom = float((ref ** 2).sum())
    nmse = float(((g - ref) ** 2).sum()) / denom if denom > 0 else 0.0
    assert nmse < NMSE_BAR, "%s: NMSE %.3g" % (what, nmse)
    return {"max_abs": float(err.max()) if err.size else 0.0, "nmse": nmse}


def assert_bf16_close_or_tie(got: torch.Tensor, ref: np.ndarray, ties: np.ndarray,
                             what: str = "") -> dict:
    """As assert_bf16_close, for the rounding contracts that round the
    normalised value to bf16 before the rotation: an element may miss the
    tolerance only where the oracle marks it as depending on a value within
    1e-3 bf16 quanta of a rounding midpoint (there the kernel's fp32 rsqrt and
    sum of squares may round to the other neighbour, one quantum away)."""
    g = bf16_to_f64(got).reshape(ref.shape)
    err = np.abs(g - ref)
    bound = BF16_ATOL + BF16_RTOL * np.abs(ref)
    bad = ~(err <= bound)
    unexplained = bad & ~ties
    if unexplained.any():
        idx = np.argwhere(unexplained)[:5]
        rows = ["%s: got %r ref %r" % (tuple(i), g[tuple(i)], ref[tuple(i)]) for i in idx]
        raise AssertionError("%s: %d of %d outside |err| <= 1e-2 + 1.6e-2|ref| away from a "
                             "rounding tie; first: %s" % (what, int(unexplained.sum()), bad.size,
                                                          "; ".join(rows)))
    denom = float((ref ** 2).sum())
    nmse = float(((g - ref) ** 2).sum()) / denom if denom > 0 else 0.0
    assert nmse < NMSE_BAR, "%s: NMSE %.3g" % (what, nmse)
    return {"max_abs": float(err.max()) if err.size else 0.0, "nmse": nmse,
            "tie_elements": int(ties.sum()), "outside_at_ties": int(bad.sum())}


def assert_plane_close(got: np.ndarray, ref: np.ndarray, mask: np.ndarray, what: str = ""):
    g = got[mask].astype(np.float64)
    r = ref[mask].astype(np.float64)
    bad = ~(np.abs(g - r) <= PLANE_RTOL * np.abs(r))
    if bad.any():
        i = np.argmax(bad)
        raise AssertionError("%s: %d of %d planes cells beyond 2e-6 relative; e.g. got %r ref %r"
                             % (what, int(bad.sum()), bad.size, g[i], r[i]))


class Guarded:
    """A device buffer with sentinel guard bands before and after the payload."""

    def __init__(self, shape, dtype=torch.bfloat16, guard: int = 4096, fill_payload=True):
        self.shape = tuple(shape)
        self.dtype = dtype
        n = int(np.prod(self.shape)) if self.shape else 1
        self.n, self.guard = n, guard
        self.ibits = torch.int16 if dtype == torch.bfloat16 else torch.int32
        pattern = SENTINEL_BF16 if dtype == torch.bfloat16 else SENTINEL_F32
        if self.ibits == torch.int32 and pattern >= 2 ** 31:
            pattern -= 2 ** 32
        self.pattern = pattern
        self.buf = torch.full((guard + n + guard,), pattern, dtype=self.ibits, device="cuda")
        self.tensor = self.buf[guard:guard + n].view(dtype).view(self.shape)

    def check(self):
        head = self.buf[:self.guard]
        tail = self.buf[self.guard + self.n:]
        assert bool((head == self.pattern).all()), "write before the output buffer"
        assert bool((tail == self.pattern).all()), "write past the output buffer"

    def untouched(self) -> np.ndarray:
        """Mask of payload cells still holding the sentinel."""
        return (self.buf[self.guard:self.guard + self.n] == self.pattern).cpu().numpy().reshape(self.shape)
