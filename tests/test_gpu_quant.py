"""GPU parity of the FP8 quantisers (fp8g_quantize_1x128 / _128x128, through
the C ABI) against the CPU oracle's quantiser: codes and scales must match bit
for bit (both sides take the rounding decisions in FP32, the precision the
scale and the quotient are defined in).  Inputs are drawn by the seeded
generator (bf16 values, and float32 values with x50 outlier groups as in the
large dense workload); edge cases: all-zero groups, ragged row counts, a
partial last 128-row block of the weights, rounding midpoints, huge and
subnormal values, negative zero."""
import numpy as np
import pytest
import torch

import oracle
from fp8_block_scaled_x128_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from fp8_block_scaled_x128_b200 import gemm
    return gemm


def draw(seed, rows, K, sigma=1.0, outlier_frac=0.0):
    """bf16 values (as float32) from the generator's normal stream; outlier
    groups multiplied by 50 in float32 (then no longer bf16)."""
    x = synth.round_to_bf16(synth.normal(synth.stream_key(seed, 9), 0, rows * K, sigma)).reshape(rows, K)
    if outlier_frac:
        u = synth.uniform(synth.stream_key(seed, 10), 0, rows * (K // 128)).reshape(rows, K // 128)
        x = (x.reshape(rows, K // 128, 128) * np.where(u < outlier_frac, np.float32(50), np.float32(1))[:, :, None]
             ).reshape(rows, K).astype(np.float32)
    return x


def to_dev(x, dtype):
    t = torch.from_numpy(np.ascontiguousarray(x, np.float32)).cuda()
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def host(t):
    torch.cuda.synchronize()
    return t.cpu().numpy()


def check_1x128(g, x, dtype):
    rows, K = x.shape
    q, sa = g.quantize_1x128(to_dev(x, dtype))
    eq, esa = oracle.quantize_1x128(x, ld_sa=sa.shape[1])
    assert np.array_equal(host(sa)[:, :rows], esa[:, :rows])
    got = host(q)
    bad = np.argwhere(got != eq)
    assert bad.size == 0, f"{len(bad)} codes differ, first at {bad[0]}: gpu {got[tuple(bad[0])]:#x} oracle " \
                          f"{eq[tuple(bad[0])]:#x} x={x[tuple(bad[0])]!r}"


def check_128x128(g, x, dtype):
    q, sb = g.quantize_128x128(to_dev(x, dtype))
    eq, esb = oracle.quantize_128x128(x)
    assert np.array_equal(host(sb), esb)
    got = host(q)
    bad = np.argwhere(got != eq)
    assert bad.size == 0, f"{len(bad)} codes differ, first at {bad[0]}: gpu {got[tuple(bad[0])]:#x} oracle {eq[tuple(bad[0])]:#x}"


@pytest.mark.parametrize("rows,K", [(1, 128), (37, 384), (256, 7168), (4097, 1024)])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_quantize_1x128_matches_oracle(g, rows, K, dtype):
    x = draw(rows + K, rows, K, outlier_frac=0.05 if dtype == "f32" else 0.0)
    if rows > 3:
        x[3, :128] = 0.0                       # an all-zero group
        x[2, :64] = -0.0                       # negative zeros
    check_1x128(g, x, dtype)


def test_quantize_1x128_rounding_midpoints_and_extremes(g):
    # rows whose quotients x/scale land on e4m3 rounding midpoints, near the
    # saturation limit, in the subnormal range, and with a huge or tiny amax
    K = 128
    mids = []
    for c in range(0, 0x7E):
        lo, hi = oracle.e4m3_value(c), oracle.e4m3_value(c + 1)
        mids.append((lo + hi) / 2)
    rows = []
    for start in range(0, len(mids), 127):
        r = np.zeros(K, np.float32)
        chunk = np.array(mids[start:start + 127], np.float32)
        r[:len(chunk)] = chunk
        r[127] = 448.0                       # amax = 448 -> scale = 1, quotients exact
        rows.append(r)
        rows.append(-r)
    rows.append(np.linspace(-3e38, 3e38, K).astype(np.float32))
    rows.append((np.arange(K) - 64).astype(np.float32) * np.float32(1e-40))   # float32 subnormals
    x = np.stack(rows).astype(np.float32)
    check_1x128(g, x, "f32")


@pytest.mark.parametrize("N,K", [(128, 128), (2112, 512), (200, 7168), (64, 256)])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_quantize_128x128_matches_oracle(g, N, K, dtype):
    x = draw(N * 3 + K, N, K, sigma=0.02)
    x[:min(N, 128), :128] = 0.0                # an all-zero block
    check_128x128(g, x, dtype)


def test_quantized_operands_feed_the_gemm(g):
    """Quantise bf16 activations and weights on the GPU, run the dense GEMM on
    the codes and scales, and compare with the oracle GEMM over the oracle's
    quantisation of the same values: identical codes and scales give the same
    product within the GEMM tolerance."""
    from .parity_util import assert_close
    M, N, K = 96, 264, 1024
    xa, xb = draw(1, M, K), draw(2, N, K, sigma=0.02)
    qa, sa = g.quantize_1x128(to_dev(xa, "bf16"))
    qb, sb = g.quantize_128x128(to_dev(xb, "bf16"))
    D = g.fp8_gemm_nt(qa, sa, qb, sb)
    eqa, esa = oracle.quantize_1x128(xa)
    eqb, esb = oracle.quantize_128x128(xb)
    ex, _ = oracle.gemm_nt(eqa, esa, esa.shape[1], eqb, esb, M, N, K)
    torch.cuda.synchronize()
    assert_close(D.view(torch.int16).cpu().numpy().view(np.uint16), ex, "quantise -> GEMM")
