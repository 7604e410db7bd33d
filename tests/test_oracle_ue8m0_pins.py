"""Pins of the oracle's power-of-two-scale GEMM (oracle.c:
fp8o_ue8m0_value, fp8o_gemm_nt_ue8m0): the E8M0 decode against its
definition (2^(e-127), 255 = NaN) and numpy's ldexp; the GEMM against a
brute-force float64 product of fully dequantised operands and against exact
integer arithmetic."""
from fractions import Fraction

import numpy as np

import oracle

from .test_oracle_pins import random_codes, torch_decode


def test_ue8m0_decode():
    for e in range(255):
        assert oracle.ue8m0_value(e) == float(np.ldexp(1.0, e - 127))
    assert np.isnan(oracle.ue8m0_value(255))
    assert oracle.ue8m0_value(127) == 1.0 and oracle.ue8m0_value(0) == 2.0 ** -127


def test_ue8m0_gemm_matches_bruteforce():
    rng = np.random.default_rng(4)
    M, N, K = 37, 200, 384
    KB, NB = K // 128, (N + 127) // 128
    A, B = random_codes(rng, (M, K)), random_codes(rng, (N, K))
    ld = 40
    sfa = rng.integers(110, 145, (KB, ld)).astype(np.uint8)
    sfb = rng.integers(110, 145, (NB, KB)).astype(np.uint8)
    ex, bf = oracle.gemm_nt_ue8m0(A, sfa, ld, B, sfb, M, N, K)
    sa = np.ldexp(1.0, sfa[:, :M].astype(np.int64) - 127).T            # [M, KB]
    sb = np.ldexp(1.0, sfb.astype(np.int64) - 127)                     # [NB, KB]
    Ad = torch_decode(A) * np.repeat(sa, 128, axis=1)
    Bd = torch_decode(B) * np.repeat(sb[np.arange(N) // 128], 128, axis=1)
    ref = Ad @ Bd.T
    assert np.all(np.abs(ex - ref) <= 1e-12 * (np.abs(Ad) @ np.abs(Bd).T))


def test_ue8m0_gemm_exact():
    rng = np.random.default_rng(5)
    M, N, K = 5, 3, 256
    lut = np.array([0xC0, 0xB8, 0x00, 0x38, 0x40], np.uint8)   # -2, -1, 0, 1, 2
    ia, ib = rng.integers(0, 5, (M, K)), rng.integers(0, 5, (N, K))
    A, B = lut[ia], lut[ib]
    sfa = rng.integers(124, 131, (2, M)).astype(np.uint8)
    sfb = rng.integers(124, 131, (1, 2)).astype(np.uint8)
    ex, _ = oracle.gemm_nt_ue8m0(A, sfa, M, B, sfb, M, N, K)
    val = np.array([-2, -1, 0, 1, 2])
    for m in range(M):
        for n in range(N):
            tot = Fraction(0)
            for kb in range(2):
                part = sum(int(val[ia[m, k]] * val[ib[n, k]]) for k in range(128 * kb, 128 * kb + 128))
                tot += part * Fraction(2) ** (int(sfa[kb, m]) - 127) * Fraction(2) ** (int(sfb[0, kb]) - 127)
            assert ex[m, n] == float(tot)
