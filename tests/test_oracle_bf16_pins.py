"""Pins of the oracle's BF16 NT GEMM (oracle.c: fp8o_bf16_gemm_nt): a numpy
float64 matrix product (the library routine the definition reduces to),
exact small-integer products that must round bit for bit, and closed forms
(identity B returns A's columns; negating B negates D)."""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from fp8_block_scaled_x128_b200 import synth


def bf16_vals(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def random_bf16(seed, shape, sigma=1.0):
    return synth.bf16_bits(synth.round_to_bf16(synth.normal(synth.stream_key(seed, 20), 0, int(np.prod(shape)), sigma)
                                               .reshape(shape)))


@pytest.mark.parametrize("M,N,K", [(5, 7, 64), (33, 40, 256), (1, 128, 1000)])
def test_bf16_gemm_matches_numpy(M, N, K):
    A, B = random_bf16(M, (M, K)), random_bf16(N + 1, (N, K))
    ex, bf = oracle.bf16_gemm_nt(A, B)
    ref = bf16_vals(A) @ bf16_vals(B).T
    bound = np.abs(bf16_vals(A)) @ np.abs(bf16_vals(B)).T
    assert np.all(np.abs(ex - ref) <= 1e-12 * bound)
    assert np.array_equal(bf, np.array([[oracle.bf16_rne(v) for v in row] for row in ex], np.uint16))


def test_bf16_gemm_exact_integers():
    rng = np.random.default_rng(1)
    M, N, K = 9, 11, 300
    a = rng.integers(-8, 9, (M, K)).astype(np.float32)
    b = rng.integers(-8, 9, (N, K)).astype(np.float32)
    A, B = synth.bf16_bits(a), synth.bf16_bits(b)
    ex, bf = oracle.bf16_gemm_nt(A, B)
    for m in range(M):
        for n in range(N):
            exact = sum(Fraction(int(x)) * Fraction(int(y)) for x, y in zip(a[m], b[n]))
            assert ex[m, n] == float(exact)
    assert np.array_equal(bf, synth.bf16_bits(synth.round_to_bf16(ex.astype(np.float32))))


def test_bf16_gemm_closed_forms():
    M, K = 6, 64
    A = random_bf16(3, (M, K))
    I = synth.bf16_bits(np.eye(K, dtype=np.float32))
    ex, bf = oracle.bf16_gemm_nt(A, I)
    assert np.array_equal(bf, A)
    B = random_bf16(4, (5, K))
    ex1, _ = oracle.bf16_gemm_nt(A, B)
    ex2, _ = oracle.bf16_gemm_nt(A, B ^ np.uint16(0x8000))
    assert np.array_equal(ex2, -ex1)
    sub = np.array([4, 0], np.int32)
    ex3, _ = oracle.bf16_gemm_nt(A, B, rows=sub)
    assert np.array_equal(ex3, ex1[sub])
