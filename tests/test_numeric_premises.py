"""Arithmetic facts the kernels rely on, checked on the host in IEEE fp32.

The assignment kernel builds its candidate masks from the sign bit of the
rounded difference w - t instead of comparing w >= t: under round-to-nearest
the sign of a rounded difference of two finite floats is the sign of the
exact difference, and equal operands give +0, except -0 - (+0) = -0, which
the kernel avoids by taking a zero threshold as -0.  The same holds for
w = -inf (the padding columns) against a finite threshold.
"""
from __future__ import annotations

import numpy as np


def _sign_clear(w: np.ndarray, t: np.ndarray) -> np.ndarray:
    t = t.astype(np.float32)
    t = np.where(t == 0, np.float32(-0.0), t).astype(np.float32)  # a zero threshold as -0
    d = (w.astype(np.float32) - t).astype(np.float32)
    return (d.view(np.uint32) >> np.uint32(31)) == 0


def test_plain_difference_misses_minus_zero_against_plus_zero():
    # the reason for the -0 threshold: without it, -0 >= +0 would be missed
    d = (np.float32(-0.0) - np.float32(0.0)).astype(np.float32)
    assert (d.view(np.uint32) >> np.uint32(31)) == 1
    assert np.float32(-0.0) >= np.float32(0.0)


def test_sign_of_rounded_difference_decides_ge_random():
    rng = np.random.default_rng(7)
    w = rng.standard_normal(200_000).astype(np.float32) * np.float32(50)
    # thresholds next to the values: equal, one ulp either side, and random
    t = np.concatenate([
        w,
        np.nextafter(w, np.float32(np.inf)),
        np.nextafter(w, np.float32(-np.inf)),
        rng.standard_normal(200_000).astype(np.float32) * np.float32(50),
    ])
    ww = np.concatenate([w, w, w, w])
    assert np.array_equal(_sign_clear(ww, t), ww >= t)


def test_sign_of_rounded_difference_decides_ge_edges():
    f = np.float32
    big = np.finfo(np.float32).max
    tiny = np.finfo(np.float32).smallest_subnormal
    cases = [
        (f(0.0), f(0.0)), (f(-0.0), f(0.0)), (f(0.0), f(-0.0)), (f(-0.0), f(-0.0)),
        (f(tiny), f(0.0)), (f(0.0), f(tiny)), (f(-tiny), f(0.0)),
        (f(big), f(-big)), (f(-big), f(big)), (f(big), f(big)),
        (f(-np.inf), f(-big)), (f(-np.inf), f(0.0)), (f(1.0), f(-np.inf)),
        (f(3.0), f(3.0)), (f(-7.5), f(-7.5)),
    ]
    w = np.array([a for a, _ in cases], dtype=np.float32)
    t = np.array([b for _, b in cases], dtype=np.float32)
    with np.errstate(over="ignore", invalid="ignore"):
        got = _sign_clear(w, t)
    assert np.array_equal(got, w >= t), list(zip(w, t, got, w >= t))


def test_funnel_shift_accumulation_orders_bits():
    # (acc << 1) | (d >> 31), applied to entries 15..0, leaves entry i's sign
    # bit in bit i; the complement is the ">= threshold" mask
    rng = np.random.default_rng(11)
    w = rng.standard_normal(32).astype(np.float32)
    t = np.float32(0.1)
    d = (w - t).astype(np.float32).view(np.uint32)
    lo = hi = 0
    for i in range(15, -1, -1):
        lo = ((lo << 1) | int(d[i] >> 31)) & 0xFFFFFFFF
        hi = ((hi << 1) | int(d[i + 16] >> 31)) & 0xFFFFFFFF
    mask = ~(lo | (hi << 16)) & 0xFFFFFFFF
    want = sum(1 << i for i in range(32) if w[i] >= t)
    assert mask == want
