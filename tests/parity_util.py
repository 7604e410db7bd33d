"""Shared helpers of the parity tests: device upload of generator outputs,
the acceptance tolerance, exact-integer inputs and canary fills."""
from __future__ import annotations

import numpy as np

# Acceptance (per element, against the oracle's unrounded FP64 value):
#   |gpu - ref| <= 8e-3*|ref| + 1e-3*rms(ref)
# and globally 1 - 2<x,y>/(|x|^2 + |y|^2) < 1e-5.  The bf16 rounding of the
# output alone is up to 2^-9 = 1.95e-3 relative; FP32 accumulation over
# <= 512 K-blocks adds far less.
REL_TOL, RMS_TOL, GLOBAL_TOL = 8e-3, 1e-3, 1e-5

CANARY = 0xDEAD  # bf16 bit pattern written to D before a call where rows must stay untouched


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def assert_close(gpu_bits: np.ndarray, ref: np.ndarray, what: str = "") -> dict:
    g = bf16_to_f64(gpu_bits).ravel()
    r = np.asarray(ref, np.float64).ravel()
    assert g.shape == r.shape
    if r.size == 0:
        return {}
    rms = float(np.sqrt(np.mean(r * r)))
    err = np.abs(g - r)
    lim = REL_TOL * np.abs(r) + RMS_TOL * rms
    bad = ~(err <= lim)
    if bad.any():
        i = int(np.argmax(bad))
        raise AssertionError(f"{what}: {int(bad.sum())}/{r.size} elements out of tolerance; "
                             f"first at flat {i}: gpu={g[i]!r} ref={r[i]!r} lim={lim[i]!r}")
    den = float(np.dot(g, g) + np.dot(r, r))
    dev = 1.0 - 2.0 * float(np.dot(g, r)) / den if den > 0 else 0.0
    assert dev < GLOBAL_TOL, f"{what}: global deviation {dev}"
    return dict(max_rel=float(np.max(err / np.maximum(np.abs(r), 1e-30))), global_dev=dev)


_INT_LUT = np.array([0xC0, 0xB8, 0x00, 0x38, 0x40], np.uint8)  # e4m3 codes of -2,-1,0,1,2


def exact_integer_codes(rng, shape) -> np.ndarray:
    """e4m3 codes of integers in {-2..2}."""
    return _INT_LUT[rng.integers(0, 5, size=shape)]


def pow2_scales(rng, shape, lo=-3, hi=2) -> np.ndarray:
    """Power-of-two FP32 scales.  With |codes| <= 2 every K-block partial is an
    integer below 2^10, and every product partial*sa*sb is exact in FP32; the
    running sums stay exact while K/128 * 512 * 2^(2*hi) is below 2^24."""
    return np.ldexp(1.0, rng.integers(lo, hi + 1, size=shape)).astype(np.float32)
