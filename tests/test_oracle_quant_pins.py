"""Pins of the oracle's FP8 quantiser (oracle.c: fp8o_e4m3_encode,
fp8o_quantize_1x128, fp8o_quantize_128x128) against things other than
itself.

The quantiser is the step the pages leave to the caller (kakushin.no, "Hvorfor
FP8 og FP4 er interessant"); its granularity is the GEMM's (one FP32 scale per
1x128 row group of A, per 128x128 block of B).  Pins: torch's own float ->
float8_e4m3fn conversion (round to nearest even) and float32 division,
the round trip of every finite e4m3 code through the independently pinned
decoder, rounding midpoints and saturation from the format definition, the
generator's separately written numpy encoder, the dequantisation error bound,
and the group / block locality of the scales.
"""
import numpy as np
import pytest
import torch

import oracle
from fp8_block_scaled_x128_b200 import synth

E4M3_MAX = 448.0


def torch_codes(v_f32: np.ndarray) -> np.ndarray:
    """torch's float32 -> e4m3fn codes (RNE; callers keep |v| <= 464 so that
    torch's non-saturating conversion and saturation agree)."""
    t = torch.from_numpy(np.ascontiguousarray(v_f32, np.float32)).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy()


def encode_many(v):
    return np.array([oracle.e4m3_encode(float(x)) for x in np.asarray(v, np.float32).ravel()], np.uint8)


def finite_codes():
    return [c for c in range(256) if (c & 0x7F) != 0x7F]


def test_encode_round_trips_every_finite_code():
    for c in finite_codes():
        v = oracle.e4m3_value(c)
        assert oracle.e4m3_encode(v) == c, hex(c)


def test_encode_midpoints_round_to_even_and_saturate():
    # consecutive positive codes c, c+1: the midpoint goes to the even mantissa,
    # anything a little off the midpoint goes to the nearer code
    for c in range(0, 0x7E):
        lo, hi = oracle.e4m3_value(c), oracle.e4m3_value(c + 1)
        mid = np.float32((lo + hi) / 2)          # exact in float32
        assert float(mid) == (lo + hi) / 2
        even = c if c % 2 == 0 else c + 1
        assert oracle.e4m3_encode(mid) == even, hex(c)
        assert oracle.e4m3_encode(-mid) == even | 0x80
        assert oracle.e4m3_encode(np.nextafter(mid, np.float32(0))) == c
        assert oracle.e4m3_encode(np.nextafter(mid, np.float32(1e9))) == c + 1
    for big in (448.0, 449.0, 464.0, 479.0, 480.0, 1e6, 3.0e38):
        assert oracle.e4m3_encode(big) == 0x7E
        assert oracle.e4m3_encode(-big) == 0xFE
    assert oracle.e4m3_encode(0.0) == 0x00 and oracle.e4m3_encode(-0.0) == 0x80
    assert oracle.e4m3_encode(2.0 ** -10) == 0x00          # half the smallest subnormal: tie to even (0)
    assert oracle.e4m3_encode(np.float32(2.0 ** -10 * 1.0001)) == 0x01


def test_encode_matches_torch_and_the_generator_on_random_floats():
    rng = np.random.default_rng(1)
    v = (rng.standard_normal(40000) * np.exp(rng.uniform(-12, 6, 40000))).astype(np.float32)
    v = np.clip(v, -464, 464)
    got = encode_many(v)
    assert np.array_equal(got, torch_codes(v))
    assert np.array_equal(got, synth.e4m3_encode(v))


def _draw(seed, rows, K, sigma=1.0):
    key = synth.stream_key(seed, 9)
    return synth.round_to_bf16(synth.normal(key, 0, rows * K, sigma)).reshape(rows, K)


def _decode(q):
    return torch.from_numpy(np.ascontiguousarray(q)).view(torch.float8_e4m3fn).double().numpy()


@pytest.mark.parametrize("rows,K", [(1, 128), (37, 384), (130, 256)])
def test_quantize_1x128_against_torch(rows, K):
    x = _draw(rows + K, rows, K)
    x[0, :128] *= np.float32(50.0)            # an outlier group
    if rows > 2:
        x[2, 128:256 if K > 128 else 128] = 0  # an all-zero group (when K > 128)
    q, sa = oracle.quantize_1x128(x)
    KB = K // 128
    g = x.reshape(rows, KB, 128)
    amax = np.abs(g).max(axis=2)
    s_ref = np.where(amax > 0, (amax / np.float32(448.0)).astype(np.float32), np.float32(1.0))
    assert np.array_equal(sa[:, :rows], s_ref.T)
    assert np.all(sa[:, rows:] == 0)
    quot = (torch.from_numpy(g) / torch.from_numpy(s_ref)[:, :, None]).numpy()   # float32 division
    assert np.array_equal(q.reshape(rows, KB, 128), torch_codes(quot))
    # the largest magnitude of every non-zero group maps to +-448
    idx = np.abs(g).argmax(axis=2)
    top = np.take_along_axis(q.reshape(rows, KB, 128), idx[:, :, None], 2)[:, :, 0]
    assert np.all((top & 0x7F)[amax > 0] == 0x7E)
    assert np.all(q.reshape(rows, KB, 128)[amax == 0] & 0x7F == 0)


def test_quantize_1x128_error_bound_and_locality():
    rows, K = 24, 512
    x = _draw(3, rows, K)
    q, sa = oracle.quantize_1x128(x)
    s = np.repeat(sa[:, :rows].T.astype(np.float64), 128, axis=1)
    err = np.abs(_decode(q) * s - x)
    # half a quantum: 2^-4 relative for normal codes, 2^-10 * scale in the subnormal range
    assert np.all(err <= np.abs(x) * 2.0 ** -4 + s * 2.0 ** -10 + 1e-30)
    # changing one group changes only that group's codes and scale
    x2 = x.copy()
    x2[5, 256:384] *= np.float32(3.0)
    q2, sa2 = oracle.quantize_1x128(x2)
    diff = q2 != q
    assert diff[5, 256:384].any() or not np.array_equal(sa2, sa)
    diff[5, 256:384] = False
    assert not diff.any()
    changed = sa2 != sa
    assert changed[2, 5] and changed.sum() == 1
    # rows are independent: permuting rows permutes codes and scale columns
    perm = np.random.default_rng(0).permutation(rows)
    qp, sap = oracle.quantize_1x128(x[perm])
    assert np.array_equal(qp, q[perm]) and np.array_equal(sap[:, :rows], sa[:, :rows][:, perm])


@pytest.mark.parametrize("N,K", [(128, 128), (200, 384), (64, 256)])
def test_quantize_128x128_against_torch(N, K):
    x = _draw(N * 7 + K, N, K, sigma=0.02)
    q, sb = oracle.quantize_128x128(x)
    KB, NB = K // 128, (N + 127) // 128
    for nb in range(NB):
        r0, r1 = 128 * nb, min(N, 128 * nb + 128)
        for kb in range(KB):
            blk = x[r0:r1, 128 * kb:128 * kb + 128]
            amax = np.abs(blk).max()
            s = np.float32(amax / np.float32(448.0)) if amax > 0 else np.float32(1.0)
            assert sb[nb, kb] == s
            quot = (torch.from_numpy(blk) / torch.tensor(s)).numpy()
            assert np.array_equal(q[r0:r1, 128 * kb:128 * kb + 128], torch_codes(quot))
            assert np.count_nonzero((q[r0:r1, 128 * kb:128 * kb + 128] & 0x7F) == 0x7E) >= 1


def test_quantize_128x128_block_is_shared_by_its_rows_only():
    N, K = 256, 256
    x = _draw(11, N, K)
    q, sb = oracle.quantize_128x128(x)
    x2 = x.copy()
    x2[3, 5] = np.float32(1000.0)            # new amax of block (0, 0) only
    q2, sb2 = oracle.quantize_128x128(x2)
    assert sb2[0, 0] == np.float32(1000.0 / np.float32(448.0))
    assert np.array_equal(np.delete(sb2.ravel(), 0), np.delete(sb.ravel(), 0))
    assert np.array_equal(q2[128:], q[128:]) and np.array_equal(q2[:, 128:], q[:, 128:])
    assert not np.array_equal(q2[:128, :128], q[:128, :128])
