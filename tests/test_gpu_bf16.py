"""GPU parity of the BF16 NT GEMM (bf16_gemm_nt through the C ABI) against
the CPU oracle: the GEMM tolerance on random bf16 inputs (FP32 accumulation
on the tensor cores against the oracle's FP64 sum), bit-exact on small
integers whose sums are exact in FP32, ragged M and N (tails clipped by the
direct stores and by the TMA-store epilogue), both epilogue variants."""
import numpy as np
import pytest
import torch

import oracle
from fp8_block_scaled_x128_b200 import synth

from .parity_util import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from fp8_block_scaled_x128_b200 import gemm
    gemm.device_error(clear=True)
    yield gemm
    gemm.set_variant_override(None)


def bf16_rand(seed, shape, sigma=1.0):
    return synth.bf16_bits(synth.round_to_bf16(
        synth.normal(synth.stream_key(seed, 21), 0, int(np.prod(shape)), sigma).reshape(shape)))


def run(g, A, B, variant):
    Ad = torch.from_numpy(A.view(np.int16)).cuda().view(torch.bfloat16)
    Bd = torch.from_numpy(B.view(np.int16)).cuda().view(torch.bfloat16)
    D = torch.full((A.shape[0], B.shape[0]), -7.0, dtype=torch.bfloat16, device="cuda")
    g.set_variant_override(variant)
    try:
        g.bf16_gemm_nt(Ad, Bd, D)
        assert g.last_variant() == variant
    finally:
        g.set_variant_override(None)
    torch.cuda.synchronize()
    return D.view(torch.int16).cpu().numpy().view(np.uint16)


def variants(g):
    return [i for i, n in enumerate(g.variant_names()) if n.startswith("bf16_")]


@pytest.mark.parametrize("shape", [(1, 8, 64), (256, 256, 64), (300, 520, 1024), (1000, 2056, 384), (64, 4096, 2048)],
                         ids=lambda s: "x".join(map(str, s)))
def test_bf16_matches_oracle(g, shape):
    M, N, K = shape
    A, B = bf16_rand(M + K, (M, K)), bf16_rand(N + 3, (N, K), 0.05)
    ex, _ = oracle.bf16_gemm_nt(A, B)
    for v in variants(g):
        assert_close(run(g, A, B, v), ex, f"{g.variant_names()[v]} {shape}")
    assert g.device_error() == 0


def test_bf16_exact_integers_bit_exact(g):
    rng = np.random.default_rng(2)
    M, N, K = 200, 264, 1024
    A = synth.bf16_bits(rng.integers(-4, 5, (M, K)).astype(np.float32))
    B = synth.bf16_bits(rng.integers(-4, 5, (N, K)).astype(np.float32))
    _, bf = oracle.bf16_gemm_nt(A, B)      # |sums| <= 16384: exact in FP32
    for v in variants(g):
        assert np.array_equal(run(g, A, B, v), bf), g.variant_names()[v]


@pytest.mark.slow
def test_bf16_large_sampled_rows(g):
    M, N, K = 4096, 4096, 4096
    A, B = bf16_rand(5, (M, K)), bf16_rand(6, (N, K), 0.05)
    rows = np.unique(np.r_[0, M - 1, 255, 256, np.random.default_rng(0).choice(M, 28, replace=False)]).astype(np.int32)
    ex, _ = oracle.bf16_gemm_nt(A, B, rows=rows)
    for v in variants(g):
        assert_close(run(g, A, B, v)[rows], ex, g.variant_names()[v])
