"""GPU parity of the power-of-two-scale FP8 GEMM (fp8_gemm_nt_ue8m0, the
block-scaled tensor-core MMA, through the C ABI) against the CPU oracle.
Bit-exact on integer codes with distinct power-of-two scales for every row
group, B block and K-block (this also pins the tensor-memory layout of the
scale factors: a scale applied to the wrong rows, columns or K-block changes
the result); the GEMM tolerance on N(0,1) data quantised with power-of-two
scales; ragged M and N."""
import numpy as np
import pytest
import torch

import oracle
from fp8_block_scaled_x128_b200 import synth

from .parity_util import assert_close, exact_integer_codes

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from fp8_block_scaled_x128_b200 import gemm
    gemm.device_error(clear=True)
    return gemm


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def run(g, A, sfa, B, sfb):
    D = g.fp8_gemm_nt_ue8m0(dev(A), dev(sfa), dev(B), dev(sfb))
    torch.cuda.synchronize()
    return D.view(torch.int16).cpu().numpy().view(np.uint16)


def pow2_quantise_rows(x):
    """[R, K] float32 -> codes and E8M0 exponents [R, KB]: scale 2^ceil(log2(amax/448))."""
    R, K = x.shape
    g = x.reshape(R, K // 128, 128)
    amax = np.abs(g).max(axis=2)
    e = np.where(amax > 0, np.ceil(np.log2(np.maximum(amax, 1e-30) / 448.0)), 0).astype(np.int64)
    codes = synth.e4m3_encode((g / np.ldexp(1.0, e)[:, :, None]).astype(np.float32)).reshape(R, K)
    return codes, (e + 127).astype(np.uint8)


@pytest.mark.parametrize("shape", [(128, 256, 128), (200, 520, 1024), (1, 8, 128), (129, 264, 384)],
                         ids=lambda s: "x".join(map(str, s)))
def test_ue8m0_exact_integers_bit_exact(g, shape):
    M, N, K = shape
    rng = np.random.default_rng(M + N + K)
    KB, NB = K // 128, (N + 127) // 128
    A, B = exact_integer_codes(rng, (M, K)), exact_integer_codes(rng, (N, K))
    ld = synth.ld_for(M)
    sfa = rng.integers(124, 131, (KB, ld)).astype(np.uint8)
    sfb = rng.integers(124, 131, (NB, KB)).astype(np.uint8)
    _, bf = oracle.gemm_nt_ue8m0(A, sfa, ld, B, sfb, M, N, K)
    assert np.array_equal(run(g, A, sfa, B, sfb), bf)
    assert g.device_error() == 0


@pytest.mark.parametrize("shape", [(256, 512, 1024), (300, 4096, 7168), (64, 2112, 7168)],
                         ids=lambda s: "x".join(map(str, s)))
def test_ue8m0_quantised_normal_data(g, shape):
    M, N, K = shape
    xa = synth.round_to_bf16(synth.normal(synth.stream_key(M, 30), 0, M * K)).reshape(M, K)
    xb = synth.round_to_bf16(synth.normal(synth.stream_key(N, 31), 0, N * K, 0.02)).reshape(N, K)
    A, ea = pow2_quantise_rows(xa)
    ld = synth.ld_for(M)
    sfa = np.full((K // 128, ld), 127, np.uint8)
    sfa[:, :M] = ea.T
    # B: one exponent per 128x128 block
    NB = (N + 127) // 128
    B = np.empty((N, K), np.uint8)
    sfb = np.empty((NB, K // 128), np.uint8)
    for nb in range(NB):
        blk = xb[128 * nb:128 * nb + 128].reshape(-1, K // 128, 128)
        amax = np.abs(blk).max(axis=(0, 2))
        e = np.ceil(np.log2(amax / 448.0)).astype(np.int64)
        B[128 * nb:128 * nb + 128] = synth.e4m3_encode(
            (blk / np.ldexp(1.0, e)[None, :, None]).astype(np.float32)).reshape(-1, K)
        sfb[nb] = (e + 127).astype(np.uint8)
    ex, _ = oracle.gemm_nt_ue8m0(A, sfa, ld, B, sfb, M, N, K)
    assert_close(run(g, A, sfa, B, sfb), ex, f"ue8m0 {shape}")
    assert g.device_error() == 0
