"""Pins of the oracle's expert pipeline around the contiguous grouped GEMM
(oracle.c: fp8o_moe_layout, fp8o_moe_dispatch, fp8o_moe_combine) against
independent constructions: a numpy stable sort by expert for the positions,
the layout rules of the contiguous GEMM (one expert per 128-row block, -1 for
unused blocks), the separately pinned 1x128 quantiser for the gathered rows,
and a float64 emulation of the FP32 fused multiply-add chain of the combine
(exact for the value ranges used)."""
import numpy as np
import pytest

import oracle
from fp8_block_scaled_x128_b200 import synth


def routing(seed, T, topk, G, drop=0.0):
    rng = np.random.default_rng(seed)
    e = np.stack([rng.choice(G, topk, replace=False) for _ in range(T)]).astype(np.int32).ravel()
    if drop:
        e[rng.random(e.size) < drop] = -1
    return e


def numpy_layout(e, G):
    """Positions from a stable argsort by expert plus 128-row padding."""
    valid = np.nonzero(e >= 0)[0]
    order = valid[np.argsort(e[valid], kind="stable")]
    cnt = np.bincount(e[valid], minlength=G)
    padded = (cnt + 127) // 128 * 128
    off = np.concatenate([[0], np.cumsum(padded)[:-1]])
    pos = np.full(e.size, -1, np.int64)
    start = np.concatenate([[0], np.cumsum(cnt)[:-1]])
    for i, r in enumerate(order):
        g = e[r]
        pos[r] = off[g] + (i - start[g])
    return cnt, off, pos, padded


@pytest.mark.parametrize("T,topk,G,drop", [(1, 1, 1, 0.0), (300, 2, 5, 0.0), (1000, 8, 64, 0.1), (37, 3, 4, 0.0)])
def test_layout_matches_a_stable_sort(T, topk, G, drop):
    e = routing(T + G, T, topk, G, drop)
    blocks = (e.size + 127) // 128 + G
    used, cnt, off, pos, mi = oracle.moe_layout(e, G, blocks)
    ncnt, noff, npos, padded = numpy_layout(e, G)
    assert np.array_equal(cnt, ncnt) and np.array_equal(off, noff) and np.array_equal(pos, npos)
    assert used == padded.sum() // 128
    # m_indices: expert g on its padded segment, -1 after the last one
    want = np.full(blocks, -1)
    for g in range(G):
        want[off[g] // 128:(off[g] + padded[g]) // 128] = g
    assert np.array_equal(mi, want)
    # every valid row lands in its expert's block, no two rows share a slot
    v = pos[e >= 0]
    assert len(np.unique(v)) == len(v)
    assert np.array_equal(mi[v // 128], e[e >= 0])


def test_layout_rejects_too_few_blocks():
    e = np.zeros(300, np.int32)              # 300 rows of expert 0 need 3 blocks
    with pytest.raises(ValueError):
        oracle.moe_layout(e, 1, 2)
    assert oracle.moe_layout(e, 1, 3)[0] == 3


def test_dispatch_rows_are_the_quantised_tokens_and_padding_is_zero():
    T, topk, G, K = 90, 2, 3, 384
    x = synth.round_to_bf16(synth.normal(synth.stream_key(1, 9), 0, T * K)).reshape(T, K)
    e = routing(2, T, topk, G)
    blocks = (T * topk + 127) // 128 + G
    used, A, sa, pos, mi = oracle.moe_dispatch(x, e, topk, G, blocks, fill=0xAB)
    q, s = oracle.quantize_1x128(x)
    for r in range(T * topk):
        assert np.array_equal(A[pos[r]], q[r // topk])
        assert np.array_equal(sa[:, pos[r]], s[:, r // topk])
    filled = np.zeros(blocks * 128, bool)
    filled[pos] = True
    inside = np.repeat(mi >= 0, 128)
    pad = inside & ~filled
    assert np.all(A[pad] == 0) and np.all(sa[:, pad] == 0)
    assert np.all(A[~inside] == 0xAB)          # unused blocks untouched
    # dequantised rows reproduce the tokens within half a quantum
    dec = oracle_decode(A[pos]) * np.repeat(sa[:, pos].T, 128, axis=1)
    tok = x[np.arange(T * topk) // topk]
    assert np.all(np.abs(dec - tok) <= np.abs(tok) * 2.0 ** -4 + np.repeat(sa[:, pos].T, 128, axis=1) * 2.0 ** -10)


def oracle_decode(codes):
    lut = np.array([oracle.e4m3_value(c) for c in range(256)])
    return lut[codes]


def emulate_combine(D_bits, pos, w, T, topk):
    """float64 emulation of acc = fmaf(w, d, acc) in float32: the product of a
    float32 and a bf16 value is exact in float64, and for these ranges so is
    the sum, so each step rounds once, like the fused multiply-add."""
    d = (D_bits.astype(np.uint32) << 16).view(np.float32)
    out = np.zeros((T, D_bits.shape[1]), np.float32)
    for t in range(T):
        acc = np.zeros(D_bits.shape[1], np.float32)
        for k in range(topk):
            r = t * topk + k
            if pos[r] < 0:
                continue
            wk = np.float64(1.0 if w is None else w[r])
            acc = (wk * d[pos[r]].astype(np.float64) + acc.astype(np.float64)).astype(np.float32)
        out[t] = acc
    return synth.bf16_bits(synth.round_to_bf16(out))


def test_combine_is_a_gather_for_one_slot_and_a_weighted_fma_chain():
    rng = np.random.default_rng(3)
    T, N, G = 50, 64, 4
    e = routing(4, T, 1, G)
    used, cnt, off, pos, mi = oracle.moe_layout(e, G, (T + 127) // 128 + G)
    D = synth.bf16_bits(synth.round_to_bf16(rng.standard_normal((used * 128, N)).astype(np.float32)))
    assert np.array_equal(oracle.moe_combine(D, pos, None, T, 1), D[pos])
    topk = 3
    e = routing(5, T, topk, G, drop=0.1)
    used, cnt, off, pos, mi = oracle.moe_layout(e, G, (T * topk + 127) // 128 + G)
    D = synth.bf16_bits(synth.round_to_bf16(rng.uniform(0.5, 4.0, (used * 128, N)).astype(np.float32)
                                            * rng.choice([-1, 1], (used * 128, N))))
    w = rng.uniform(0.25, 1.0, T * topk).astype(np.float32)
    got = oracle.moe_combine(D, pos, w, T, topk)
    assert np.array_equal(got, emulate_combine(D, pos, w, T, topk))


def fused_tie_cases():
    """(d, w) with w * d = 2^-8 + 2^-24 + delta, 0 < delta < 2^-32: added to 1.0
    with one rounding (a fused multiply-add) the FP32 sum lies above the bf16
    tie 1 + 2^-8 and rounds up to 1 + 2^-7 (bits 0x3F81); rounding the product
    first drops delta, the sum lands on the FP32 tie, rounds to even, and the
    bf16 result is the tie itself, which rounds down to 1.0 (0x3F80)."""
    from fractions import Fraction as F
    target = F(1, 2 ** 8) + F(1, 2 ** 24)
    out = []
    for mant in range(128):
        d = F(128 + mant, 128)                  # bf16 values in [1, 2)
        w = np.float32(float(target / d))
        if F(float(w)) < target / d:
            w = np.nextafter(w, np.float32(1))
        delta = F(float(w)) * d - target
        if 0 < delta < F(1, 2 ** 32):
            out.append((float(d), float(w)))
    return out


def test_combine_rounds_once_per_slot():
    cases = fused_tie_cases()
    assert len(cases) > 40
    T, topk, N = len(cases), 2, 8
    pos = np.arange(T * topk, dtype=np.int32)
    d = np.zeros((T * topk, N), np.float32)
    w = np.zeros(T * topk, np.float32)
    for t, (dv, wv) in enumerate(cases):
        d[2 * t], w[2 * t] = 1.0, 1.0            # slot 0: acc = 1.0
        d[2 * t + 1], w[2 * t + 1] = dv, wv     # slot 1: the crafted product
    D = synth.bf16_bits(d)
    got = oracle.moe_combine(D, pos, w, T, topk)
    assert np.all(got == 0x3F81)
    assert np.array_equal(got, emulate_combine(D, pos, w, T, topk))
