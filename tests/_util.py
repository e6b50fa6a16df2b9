"""Comparison helpers shared by the GPU parity tests (test code only)."""
import os

import numpy as np
import torch

import oracle as O

# (test, what, elements that needed the fp32 accumulation bound, elements
# checked) for every bf16 comparison; printed in the pytest terminal summary.
FALLBACK_LOG = []


def record_fallback(what: str, n_fallback: int, n_total: int):
    test = os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0]
    FALLBACK_LOG.append((test, what, int(n_fallback), int(n_total)))


def bits(t: torch.Tensor) -> np.ndarray:
    """Raw bf16 bits of a (CPU or GPU) bf16 tensor as uint16 numpy."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def from_bits(u16: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).view(torch.bfloat16)


def bf16_ordinal(u16: np.ndarray) -> np.ndarray:
    u = u16.astype(np.int32)
    return np.where(u & 0x8000, -(u & 0x7FFF), u)


def bf16_ulp(y: np.ndarray) -> np.ndarray:
    """Spacing of bf16 values at |y| (binary64)."""
    a = np.abs(y)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -126)
    return np.exp2(e - 7)


def check_bf16(y_bits: np.ndarray, Y_exact: np.ndarray, absY: np.ndarray, rel: float = 1e-5,
               what: str = "output"):
    """The tolerance of the W4A8 outputs: within 1 bf16 ulp of the correctly
    rounded exact value; where the exact value nearly cancels, the fp32
    accumulation bound |y - Y| <= rel * sum|terms| (+ the final half-ulp
    rounding) is accepted instead.  Returns the number of elements that
    needed the second bound."""
    ref = O.f64_to_bf16(Y_exact)
    d = np.abs(bf16_ordinal(y_bits) - bf16_ordinal(ref))
    y = O.bf16_to_f32(y_bits).astype(np.float64)
    fallback = np.abs(y - Y_exact) <= rel * absY + 0.5 * bf16_ulp(Y_exact) + 1e-30
    ok = (d <= 1) | fallback
    if not ok.all():
        i = np.argwhere(~ok)[:5]
        raise AssertionError(
            f"{what}: {int((~ok).sum())} / {ok.size} elements out of tolerance; first {i.tolist()}: "
            f"gpu={y[tuple(i[0])]!r} exact={Y_exact[tuple(i[0])]!r} ulps={d[tuple(i[0])]} "
            f"abs_terms={absY[tuple(i[0])]!r}")
    n = int(((d > 1) & fallback).sum())
    record_fallback(what, n, ok.size)
    return n


def to_dev(a: np.ndarray, dtype=None, device="cuda"):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.to(device)
