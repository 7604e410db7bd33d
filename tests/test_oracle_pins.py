"""Pins of the CPU oracle against things other than itself.

Each check ties the oracle to an independent source: torch's own e4m3 and
bf16 conversions, numpy float64 matrix products over fully dequantised
operands, exact integer arithmetic, hand-derived worked examples
(tests/golden/worked_examples.txt) and structural invariants of the grouped
layouts (GeekNews "DeepSeek, DeepGEMM 오픈소스 공개", MoE grouped GEMM
section).  A dropped term, a wrong scale index, a transposed operand or a
wrong rounding in the oracle fails at least one of them.
"""
import os
import re
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from fp8_block_scaled_x128_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.txt")

# ----------------------------------------------------------------------------
# independent helpers (torch decode + numpy float64 products)
# ----------------------------------------------------------------------------


def torch_decode(codes: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(codes, np.uint8)).view(torch.float8_e4m3fn)
    return t.double().numpy()


def brute_force_dense(A, sa, B, sb, M, N, K):
    """Dequantise every element with its own scale, then one float64 matmul."""
    KB = K // 128
    Ad = torch_decode(A).reshape(M, K) * np.repeat(sa[:, :M].T.astype(np.float64), 128, axis=1)
    nb = np.arange(N) // 128
    Bd = torch_decode(B).reshape(N, K) * np.repeat(sb[nb].astype(np.float64), 128, axis=1)
    ref = Ad @ Bd.T
    bound = np.abs(Ad) @ np.abs(Bd).T   # sum of |terms|: rounding-error scale
    assert Ad.shape == (M, K) and sb.shape[1] == KB
    return ref, bound


def random_codes(rng, shape):
    c = rng.integers(0, 256, size=shape, dtype=np.uint8)
    return np.where((c & 0x7F) == 0x7F, c & 0xF0, c).astype(np.uint8)   # no NaN codes


def random_scales(rng, shape):
    return (rng.uniform(0.25, 4.0, size=shape) * 2.0 ** rng.integers(-6, 6, size=shape)).astype(np.float32)


def torch_bf16_bits(x_f32: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(x_f32, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


# ----------------------------------------------------------------------------
# formats
# ----------------------------------------------------------------------------


def test_e4m3_decode_all_codes_match_torch():
    ref = torch_decode(np.arange(256, dtype=np.uint8))
    got = np.array([oracle.e4m3_value(c) for c in range(256)])
    nan = np.isnan(ref)
    assert list(np.nonzero(nan)[0]) == [0x7F, 0xFF]
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


def test_e4m3_decode_format_landmarks():
    # OCP OFP8 E4M3: bias 7, subnormal quantum 2^-9, min normal 2^-6, max 448
    assert oracle.e4m3_value(0x01) == 2.0 ** -9
    assert oracle.e4m3_value(0x07) == 7 * 2.0 ** -9
    assert oracle.e4m3_value(0x08) == 2.0 ** -6
    assert oracle.e4m3_value(0x38) == 1.0
    assert oracle.e4m3_value(0x7E) == 448.0
    assert oracle.e4m3_value(0xFE) == -448.0


def test_bf16_rne_matches_torch_on_float32_values():
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(2.0) ** rng.integers(-40, 40, 20000),
        # exact ties: a float32 whose low 16 bits are 0x8000
        (np.arange(1, 2001, dtype=np.uint32) << 16 | 0x8000).view(np.float32),
        # bf16 subnormal region
        rng.standard_normal(2000).astype(np.float32) * np.float32(2.0 ** -130),
        np.array([0.0, -0.0, 3.3895314e38, -3.3895314e38], np.float32),
    ])
    ref = torch_bf16_bits(x)
    got = np.array([oracle.bf16_rne(float(v)) for v in x], np.uint16)
    assert np.array_equal(got, ref)


def test_bf16_rne_rounds_double_once():
    # 1 + 2^-8 + 2^-40 lies just above the tie between bf16 1.0 and 1+2^-7.
    # One rounding from double gives 1+2^-7; rounding through float32 first
    # would land on the exact tie and then on 1.0.
    assert oracle.bf16_rne(1.0 + 2.0 ** -8 + 2.0 ** -40) == 0x3F81
    assert oracle.bf16_rne(1.0 + 2.0 ** -8) == 0x3F80            # tie -> even
    assert oracle.bf16_rne(1.0 + 3 * 2.0 ** -8) == 0x3F82        # tie -> even (up)
    assert oracle.bf16_rne(-(1.0 + 3 * 2.0 ** -8)) == 0xBF82
    assert oracle.bf16_rne(2.0 ** 128) == 0x7F80                 # overflow -> inf
    assert oracle.bf16_rne(2.0 ** -133) == 0x0001                # smallest subnormal
    assert oracle.bf16_rne(2.0 ** -134) == 0x0000                # tie at half quantum -> even (0)
    assert oracle.bf16_rne(1.5 * 2.0 ** -134) == 0x0001


def test_generator_e4m3_encoder_matches_torch():
    """The input generator's quantiser (not part of the oracle) agrees with torch's RNE cast."""
    rng = np.random.default_rng(2)
    x = np.concatenate([
        rng.uniform(-448, 448, 50000), rng.standard_normal(50000) * 2.0 ** rng.integers(-12, 8, 50000),
        np.array([0.0, 448.0, -448.0, 2.0 ** -9, 2.0 ** -10, 3 * 2.0 ** -11, 240.0, 232.0, 248.0]),
    ]).astype(np.float32)
    x = np.clip(x, -448, 448)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = synth.e4m3_encode(x)
    assert np.array_equal(got, ref)
    assert synth.e4m3_encode(np.array([460.0, 1e6, -1e6], np.float32)).tolist() == [0x7E, 0x7E, 0xFE]


# ----------------------------------------------------------------------------
# the GEMM definition
# ----------------------------------------------------------------------------


def _parse_golden():
    cases = []
    for line in open(GOLDEN, encoding="utf-8"):
        line = line.split("#")[0].strip()
        if not line:
            continue
        f = [p.strip() for p in line.split("|")]
        M, N, K = map(int, f[1].split())
        cases.append(dict(name=f[0], M=M, N=N, K=K, a=f[2], b=f[3], sa=f[4], sb=f[5],
                          value=float(f[6]), bits=int(f[7], 16)))
    return cases


def _fill(rule, rows, K):
    m = re.fullmatch(r"all (0x[0-9A-Fa-f]+)", rule)
    if m:
        return np.full((rows, K), int(m.group(1), 16), np.uint8)
    m = re.fullmatch(r"first (0x[0-9A-Fa-f]+) rest (0x[0-9A-Fa-f]+)", rule)
    a = np.full((rows, K), int(m.group(2), 16), np.uint8)
    a[:, 0] = int(m.group(1), 16)
    return a


def _scales(rule, KB):
    if rule.startswith("kb"):
        vals = dict(p.split(":") for p in rule.split())
        return np.array([float(vals[f"kb{k}"]) for k in range(KB)], np.float32)
    return np.full(KB, float(rule), np.float32)


@pytest.mark.parametrize("case", _parse_golden(), ids=lambda c: c["name"])
def test_worked_examples(case):
    M, N, K = case["M"], case["N"], case["K"]
    KB, NB = K // 128, (N + 127) // 128
    A, B = _fill(case["a"], M, K), _fill(case["b"], N, K)
    sa = np.repeat(_scales(case["sa"], KB)[:, None], M, axis=1)
    sb = np.repeat(_scales(case["sb"], KB)[None, :], NB, axis=0)
    ex, bf = oracle.gemm_nt(A, sa, M, B, sb, M, N, K)
    assert np.all(ex == case["value"])
    assert np.all(bf == case["bits"])


@pytest.mark.parametrize("M,N,K", [(1, 1, 128), (5, 7, 128), (17, 130, 256), (48, 40, 384), (33, 257, 256)])
def test_dense_matches_bruteforce(M, N, K):
    rng = np.random.default_rng(M * 1000 + N + K)
    KB, NB = K // 128, (N + 127) // 128
    A, B = random_codes(rng, (M, K)), random_codes(rng, (N, K))
    sa, sb = random_scales(rng, (KB, M)), random_scales(rng, (NB, KB))
    ex, bf = oracle.gemm_nt(A, sa, M, B, sb, M, N, K)
    ref, bound = brute_force_dense(A, sa, B, sb, M, N, K)
    assert np.all(np.abs(ex - ref) <= 1e-12 * bound + 1e-300)
    # the bf16 output is the one-step rounding of the exact value
    assert np.array_equal(bf, np.vectorize(oracle.bf16_rne, otypes=[np.uint16])(ex))


def test_dense_ld_sa_padding_and_row_subset():
    rng = np.random.default_rng(7)
    M, N, K, ld = 10, 20, 256, 16
    A, B = random_codes(rng, (M, K)), random_codes(rng, (N, K))
    sa = np.full((K // 128, ld), np.nan, np.float32)      # padding must never be read
    sa[:, :M] = random_scales(rng, (K // 128, M))
    sb = random_scales(rng, (1, K // 128))
    full, _ = oracle.gemm_nt(A, sa, ld, B, sb, M, N, K)
    assert np.all(np.isfinite(full))
    rows = np.array([9, 0, 4], np.int32)
    sub, _ = oracle.gemm_nt(A, sa, ld, B, sb, M, N, K, rows=rows)
    assert np.array_equal(sub, full[rows])


def test_exact_small_integers_power_of_two_scales():
    """FP8 values in {-2..2}, scales 2^e: every partial is an integer, the
    result is exact in float32, so the bf16 bits are fixed by exact math."""
    rng = np.random.default_rng(3)
    M, N, K = 24, 200, 512
    KB, NB = K // 128, 2
    lut = np.array([0xC0, 0xB8, 0x00, 0x38, 0x40], np.uint8)   # -2,-1,0,1,2
    ia, ib = rng.integers(-2, 3, (M, K)), rng.integers(-2, 3, (N, K))
    A, B = lut[ia + 2], lut[ib + 2]
    ea, eb = rng.integers(-4, 3, (KB, M)), rng.integers(-4, 3, (NB, KB))
    sa, sb = np.ldexp(1.0, ea).astype(np.float32), np.ldexp(1.0, eb).astype(np.float32)
    ex, bf = oracle.gemm_nt(A, sa, M, B, sb, M, N, K)
    exact = np.zeros((M, N), object)
    for kb in range(KB):
        p = ia[:, kb * 128:(kb + 1) * 128].astype(np.int64) @ ib[:, kb * 128:(kb + 1) * 128].T.astype(np.int64)
        for m in range(M):
            for n in range(N):
                exact[m, n] += Fraction(int(p[m, n])) * Fraction(2) ** int(ea[kb, m] + eb[n // 128, kb])
    exf = np.array([[float(v) for v in r] for r in exact])
    assert np.array_equal(ex, exf)
    assert np.array_equal(bf, torch_bf16_bits(exf.astype(np.float32)))


def test_unit_vector_b_selects_a_column():
    """B[n] = e_n (K = 128, N <= 128): D[m,n] = dec(A[m,n]) * sa[m,0] * sb[0,0]."""
    rng = np.random.default_rng(4)
    M, N, K = 16, 96, 128
    A = random_codes(rng, (M, K))
    B = np.zeros((N, K), np.uint8)
    B[np.arange(N), np.arange(N)] = 0x38
    sa, sb = random_scales(rng, (1, M)), random_scales(rng, (1, 1))
    ex, _ = oracle.gemm_nt(A, sa, M, B, sb, M, N, K)
    ref = torch_decode(A)[:, :N] * sa[0][:, None].astype(np.float64) * np.float64(sb[0, 0])
    assert np.array_equal(ex, ref)


def test_doubling_sa_row_doubles_that_row_only():
    rng = np.random.default_rng(5)
    M, N, K = 8, 150, 384
    A, B = random_codes(rng, (M, K)), random_codes(rng, (N, K))
    sa, sb = random_scales(rng, (3, M)), random_scales(rng, (2, 3))
    ex, _ = oracle.gemm_nt(A, sa, M, B, sb, M, N, K)
    sa2 = sa.copy()
    sa2[:, 3] *= 2
    ex2, _ = oracle.gemm_nt(A, sa2, M, B, sb, M, N, K)
    assert np.array_equal(ex2[3], 2 * ex[3])
    assert np.array_equal(np.delete(ex2, 3, 0), np.delete(ex, 3, 0))


def test_sb_block_boundary_uses_row_over_128():
    """Changing sb[1, kb] changes only columns n >= 128, scaled exactly."""
    rng = np.random.default_rng(6)
    M, N, K = 4, 200, 256
    A, B = random_codes(rng, (M, K)), random_codes(rng, (N, K))
    sa, sb = random_scales(rng, (2, M)), random_scales(rng, (2, 2))
    ex, _ = oracle.gemm_nt(A, sa, M, B, sb, M, N, K)
    sb2 = sb.copy()
    sb2[1, :] *= 4
    ex2, _ = oracle.gemm_nt(A, sa, M, B, sb2, M, N, K)
    assert np.array_equal(ex2[:, :128], ex[:, :128])
    assert np.array_equal(ex2[:, 128:], 4 * ex[:, 128:])


# ----------------------------------------------------------------------------
# grouped layouts
# ----------------------------------------------------------------------------


def test_contiguous_matches_bruteforce_per_expert_and_skips_minus_one():
    rng = np.random.default_rng(8)
    G, N, K = 3, 136, 256
    d = synth.contiguous_inputs(11, [100, 256, 20], N, K, empty_blocks=(1, 4))
    m_idx, M = d["m_indices"], d["M"]
    assert list(m_idx) == [0, -1, 1, 1, -1, 2]
    canary = np.full((M, N), 12345.0)
    ex, bf = oracle.m_grouped_contiguous(d["A"], d["sa"], d["ld_sa"], d["B"], d["sb"], m_idx, M, N, K, G,
                                         out_exact=canary.copy(), out_bf16=np.full((M, N), 0xBEEF, np.uint16))
    for r, g in enumerate(m_idx):
        rows = slice(128 * r, 128 * r + 128)
        if g < 0:
            assert np.all(ex[rows] == 12345.0) and np.all(bf[rows] == 0xBEEF)
            continue
        ref, bound = brute_force_dense(d["A"][rows], d["sa"][:, 128 * r:128 * r + 128], d["B"][g], d["sb"][g],
                                       128, N, K)
        assert np.all(np.abs(ex[rows] - ref) <= 1e-12 * bound + 1e-300)
    del rng


def test_contiguous_padding_rows_do_not_affect_other_rows():
    d = synth.contiguous_inputs(12, [70, 130], 64, 128)
    args = (d["ld_sa"], d["B"], d["sb"], d["m_indices"], d["M"], d["N"], d["K"], d["G"])
    ex, _ = oracle.m_grouped_contiguous(d["A"], d["sa"], *args)
    A2 = d["A"].copy()
    A2[70:128] = 0x40          # rewrite expert 0's padding rows
    A2[128 + 130:] = 0xC0      # and expert 1's
    ex2, _ = oracle.m_grouped_contiguous(A2, d["sa"], *args)
    real = np.r_[0:70, 128:128 + 130]
    assert np.array_equal(ex[real], ex2[real])


def test_masked_rows_beyond_mask_untouched_and_valid_rows_match_bruteforce():
    G, Mmax, N, K = 4, 40, 72, 256
    d = synth.masked_inputs(13, G, Mmax, N, K, masked_m=[0, 1, 39, 40])
    can_e = np.full((G, Mmax, N), -7.0)
    can_b = np.full((G, Mmax, N), 0xDEAD, np.uint16)
    ex, bf = oracle.m_grouped_masked(d["A"], d["sa"], d["ld_sa"], d["B"], d["sb"], d["masked_m"],
                                     G, Mmax, N, K, out_exact=can_e, out_bf16=can_b)
    for g, mg in enumerate(d["masked_m"]):
        assert np.all(ex[g, mg:] == -7.0) and np.all(bf[g, mg:] == 0xDEAD)
        if mg:
            ref, bound = brute_force_dense(d["A"][g, :mg], d["sa"][g][:, :mg], d["B"][g], d["sb"][g], mg, N, K)
            assert np.all(np.abs(ex[g, :mg] - ref) <= 1e-12 * bound + 1e-300)


def test_masked_group_permutation_and_independence():
    G, Mmax, N, K = 5, 24, 40, 128
    d = synth.masked_inputs(14, G, Mmax, N, K, masked_m=[24, 3, 0, 17, 9])
    run = lambda A, sa, B, sb, mm: oracle.m_grouped_masked(A, sa, d["ld_sa"], B, sb, mm, G, Mmax, N, K)[0]
    base = run(d["A"], d["sa"], d["B"], d["sb"], d["masked_m"])
    perm = np.array([3, 0, 4, 1, 2])
    permuted = run(d["A"][perm], d["sa"][perm], d["B"][perm], d["sb"][perm], d["masked_m"][perm])
    assert np.array_equal(permuted, base[perm])
    B2 = d["B"].copy()
    B2[3] = random_codes(np.random.default_rng(0), B2[3].shape)
    changed = run(d["A"], d["sa"], B2, d["sb"], d["masked_m"])
    assert not np.array_equal(changed[3, :17], base[3, :17])
    assert np.array_equal(np.delete(changed, 3, 0), np.delete(base, 3, 0))


def test_masked_over_mmax_is_clamped():
    G, Mmax, N, K = 2, 16, 16, 128
    d = synth.masked_inputs(15, G, Mmax, N, K, masked_m=[16, 16])
    full = oracle.m_grouped_masked(d["A"], d["sa"], d["ld_sa"], d["B"], d["sb"], [16, 16], G, Mmax, N, K)[0]
    over = oracle.m_grouped_masked(d["A"], d["sa"], d["ld_sa"], d["B"], d["sb"], [99, 16], G, Mmax, N, K)[0]
    assert np.array_equal(full, over)
