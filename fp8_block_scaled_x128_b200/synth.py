"""Seeded synthetic inputs for the fine-grained-scaled FP8 GEMM.

This module serves both the CUDA path and the CPU oracle with identical
inputs.  It holds none of the GEMM's arithmetic: it draws values, rounds them
to bf16, and quantises them to e4m3 codes with one FP32 scale per 1x128 group
of A and per 128x128 block of B.  That quantisation is the caller's job, not
the library's (kakushin.no, "Hvorfor FP8 og FP4 er interessant": the user
converts inputs to FP8 and transposes them), so it lives here as input
preparation.

Recipe (the same for every tensor):
  * counter-based splitmix64 stream per (seed, tensor id); element i of a
    tensor uses counters 2*(i//2) and 2*(i//2)+1;
  * uniforms u = ((z >> 11) + 0.5) * 2**-53, in (0, 1);
  * Box-Muller: r = sqrt(-2 ln u1), value = r*cos(2 pi u2) for even i,
    r*sin(2 pi u2) for odd i; times sigma; float64 -> float32 -> bf16 (RNE);
  * group amax over |x| (float32), scale = amax / 448 in float32
    (scale = 1 where amax == 0), code = e4m3_rne_satfinite(x / scale) with the
    division in float32.

Layouts produced (they are the library's boundary layouts):
  A  [rows, K] uint8 e4m3 codes, K contiguous
  sa [KB, ld_sa] float32, "MN-major": sa[kb, m] scales A[m, 128kb:128kb+128]
  B  [N, K] uint8 e4m3 codes
  sb [NB, KB] float32 row-major: sb[nb, kb] scales B[128nb:128nb+128, 128kb:...]
Grouped variants stack a leading G axis on A/sa (masked) and on B/sb.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_U64 = np.uint64
_GOLDEN = _U64(0x9E3779B97F4A7C15)
_MIX1 = _U64(0xBF58476D1CE4E5B9)
_MIX2 = _U64(0x94D049BB133111EB)
E4M3_MAX = 448.0

# tensor ids (streams) used by the workload builders
STREAM_A, STREAM_B, STREAM_OUTLIER, STREAM_MASK, STREAM_MISC = 1, 2, 3, 4, 5


def _mix(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> _U64(30))) * _MIX1
    z = (z ^ (z >> _U64(27))) * _MIX2
    return z ^ (z >> _U64(31))


def stream_key(seed: int, stream: int) -> np.uint64:
    """Base key of one tensor's counter stream."""
    with np.errstate(over="ignore"):
        s = np.array([(int(seed) * 0x100000001B3 + int(stream) * 0x2545F4914F6CDD1D) % (1 << 64)],
                     dtype=_U64)
        return _mix(s + _GOLDEN)[0]


def uniform(key: np.uint64, start: int, count: int) -> np.ndarray:
    """count uniforms in (0,1) from counters start..start+count-1 (float64)."""
    ctr = np.arange(start, start + count, dtype=_U64)
    with np.errstate(over="ignore"):
        z = _mix(key + (ctr + _U64(1)) * _GOLDEN)
    return ((z >> _U64(11)).astype(np.float64) + 0.5) * (2.0 ** -53)


def normal(key: np.uint64, start: int, count: int, sigma: float = 1.0) -> np.ndarray:
    """Elements start..start+count-1 of a N(0, sigma^2) stream (float64)."""
    if count <= 0:
        return np.zeros(0, np.float64)
    p0 = start // 2
    p1 = (start + count + 1) // 2
    u = uniform(key, 2 * p0, 2 * (p1 - p0)).reshape(-1, 2)
    r = np.sqrt(-2.0 * np.log(u[:, 0]))
    th = 2.0 * np.pi * u[:, 1]
    z = np.empty(2 * (p1 - p0), np.float64)
    z[0::2] = r * np.cos(th)
    z[1::2] = r * np.sin(th)
    off = start - 2 * p0
    return z[off:off + count] * sigma


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """float64/float32 -> float32 holding the nearest bf16 (RNE; via float32)."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    bias = _U64(0x7FFF) + ((u >> _U64(16)) & _U64(1))
    u = ((u + bias) & _U64(0xFFFF0000)).astype(np.uint32)
    return u.view(np.float32)


def bf16_bits(x_bf16_as_f32: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(x_bf16_as_f32, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """float32 -> e4m3 (OCP "fn": no inf, S.1111.111 = NaN) codes, RNE, saturating
    to +-448.  Finite inputs only."""
    x = np.asarray(x, dtype=np.float32)
    a = np.abs(x).astype(np.float64)
    sign = np.signbit(x).astype(np.uint8) << 7
    _, E = np.frexp(a)                       # a = f * 2**E, f in [0.5, 1)
    e = np.maximum(E.astype(np.int64) - 1, -6)  # unbiased exponent, subnormals at -6
    e = np.minimum(e, 8)
    q = np.ldexp(1.0, (e - 3).astype(np.int32))  # quantum: 3 mantissa bits
    n = np.rint(a / q)                       # ties to even
    up = n >= 16                             # mantissa carried into the exponent
    e = np.where(up, e + 1, e)
    n = np.where(up, n / 2, n)
    over = (e > 8) | ((e == 8) & (n > 14))    # beyond 448 -> saturate
    e = np.where(over, 8, e)
    n = np.where(over, 14, n).astype(np.int64)
    sub = n < 8                              # only reachable at e == -6
    expf = np.where(sub, 0, e + 7)
    mant = np.where(sub, n, n - 8)
    code = (expf << 3) | mant
    return (code.astype(np.uint8) | sign).astype(np.uint8)


def _scale_of(amax: np.ndarray) -> np.ndarray:
    amax = amax.astype(np.float32)
    s = amax / np.float32(E4M3_MAX)
    return np.where(amax > 0, s, np.float32(1.0)).astype(np.float32)


def quantize_rows_1x128(x: np.ndarray):
    """x [R, K] float32 (K % 128 == 0) -> codes [R, K] uint8, scale [R, KB] float32."""
    R, K = x.shape
    KB = K // 128
    xg = x.reshape(R, KB, 128)
    scale = _scale_of(np.abs(xg).max(axis=2) if R else np.zeros((0, KB), np.float32))
    codes = e4m3_encode((xg / scale[:, :, None]).astype(np.float32)).reshape(R, K)
    return codes, scale


def quantize_block_128x128(x: np.ndarray):
    """x [r<=128, K] float32 -> codes [r, K], scale [KB] float32 (one block row)."""
    r, K = x.shape
    KB = K // 128
    xg = x.reshape(r, KB, 128)
    scale = _scale_of(np.abs(xg).max(axis=(0, 2)))
    codes = e4m3_encode((xg / scale[None, :, None]).astype(np.float32)).reshape(r, K)
    return codes, scale


def _parallel(fn, items) -> None:
    """Run fn over independent chunks on a thread pool (numpy releases the GIL);
    every chunk writes a disjoint slice, so the result is the same for any
    number of threads."""
    items = list(items)
    n = min(len(items), max(1, len(os.sched_getaffinity(0))), 32)
    if n <= 1:
        for it in items:
            fn(it)
        return
    with ThreadPoolExecutor(n) as ex:
        for _ in ex.map(fn, items):
            pass


def ld_for(m: int) -> int:
    """Pitch (in floats) of one K-block row of sa: M rounded up to 4 (16 bytes)."""
    return max(4, (m + 3) // 4 * 4)


def make_a(seed: int, rows: int, K: int, sigma: float = 1.0, outlier_frac: float = 0.0,
           outlier_mult: float = 50.0, stream: int = STREAM_A, ld_sa: int | None = None,
           chunk_rows: int = 512):
    """Activations: A [rows, K] e4m3 codes and sa [KB, ld_sa] (MN-major).

    outlier_frac > 0 multiplies that fraction of 1x128 groups (chosen by a
    separate seeded stream) by outlier_mult before quantisation."""
    KB = K // 128
    ld = ld_for(rows) if ld_sa is None else ld_sa
    key = stream_key(seed, stream)
    okey = stream_key(seed, STREAM_OUTLIER)
    A = np.empty((rows, K), np.uint8)
    sa = np.zeros((KB, ld), np.float32)

    def chunk(r0):
        r1 = min(rows, r0 + chunk_rows)
        x = round_to_bf16(normal(key, r0 * K, (r1 - r0) * K, sigma)).reshape(r1 - r0, K)
        if outlier_frac > 0:
            u = uniform(okey, r0 * KB, (r1 - r0) * KB).reshape(r1 - r0, KB)
            mult = np.where(u < outlier_frac, np.float32(outlier_mult), np.float32(1.0))
            x = (x.reshape(r1 - r0, KB, 128) * mult[:, :, None].astype(np.float32)).reshape(r1 - r0, K)
        codes, sc = quantize_rows_1x128(x)
        A[r0:r1] = codes
        sa[:, r0:r1] = sc.T

    _parallel(chunk, range(0, rows, chunk_rows))
    return A, sa


def make_b(seed: int, N: int, K: int, sigma: float = 1.0, stream: int = STREAM_B):
    """Weights: B [N, K] e4m3 codes and sb [NB, KB] per 128x128 block."""
    KB = K // 128
    NB = (N + 127) // 128
    key = stream_key(seed, stream)
    B = np.empty((N, K), np.uint8)
    sb = np.empty((NB, KB), np.float32)

    def chunk(nb):
        r0, r1 = nb * 128, min(N, nb * 128 + 128)
        x = round_to_bf16(normal(key, r0 * K, (r1 - r0) * K, sigma)).reshape(r1 - r0, K)
        B[r0:r1], sb[nb] = quantize_block_128x128(x)

    _parallel(chunk, range(NB))
    return B, sb


# ---------------------------------------------------------------------------
# Workloads (the five configurations plus small parity shapes)
# ---------------------------------------------------------------------------

def dense_inputs(seed: int, M: int, N: int, K: int, a_sigma: float = 1.0, b_sigma: float = 1.0,
                 outlier_frac: float = 0.0):
    A, sa = make_a(seed, M, K, a_sigma, outlier_frac)
    B, sb = make_b(seed, N, K, b_sigma)
    return dict(A=A, sa=sa, ld_sa=sa.shape[1], B=B, sb=sb, M=M, N=N, K=K)


def grouped_b(seed: int, G: int, N: int, K: int, sigma: float = 1.0):
    """B [G, N, K] and sb [G, NB, KB]; group g uses stream STREAM_B + 16*g."""
    Bs, sbs = [], []
    for g in range(G):
        B, sb = make_b(seed, N, K, sigma, stream=STREAM_B + 16 * g)
        Bs.append(B)
        sbs.append(sb)
    return np.stack(Bs), np.stack(sbs)


def contiguous_inputs(seed: int, group_rows, N: int, K: int, empty_blocks=(), sigma: float = 1.0):
    """M-grouped contiguous layout.

    group_rows[g] = number of real rows of expert g; each expert's segment is
    padded up to a multiple of 128 rows and the segments are concatenated.
    m_indices[r] is the expert of 128-row block r.  empty_blocks inserts
    blocks marked -1 (skipped; their D rows stay untouched) before the listed
    block positions of the final layout.
    """
    G = len(group_rows)
    m_idx = []
    for g, rows in enumerate(group_rows):
        m_idx += [g] * ((rows + 127) // 128)
    for pos in sorted(empty_blocks):
        m_idx.insert(pos, -1)
    m_indices = np.array(m_idx, np.int32)
    M = 128 * len(m_indices)
    A, sa = make_a(seed, M, K)
    B, sb = grouped_b(seed, G, N, K, sigma)
    return dict(A=A, sa=sa, ld_sa=sa.shape[1], B=B, sb=sb, m_indices=m_indices,
                M=M, N=N, K=K, G=G)


def masked_m_draw(seed: int, G: int, Mmax: int) -> np.ndarray:
    """masked_m[g] ~ Uniform{0..Mmax} from the seed."""
    u = uniform(stream_key(seed, STREAM_MASK), 0, G)
    return np.minimum(np.floor(u * (Mmax + 1)), Mmax).astype(np.int32)


def masked_inputs(seed: int, G: int, Mmax: int, N: int, K: int, masked_m=None, sigma: float = 1.0):
    """M-grouped masked layout: A [G, Mmax, K], sa [G, KB, ld_sa], B [G, N, K],
    sb [G, NB, KB], masked_m [G] int32."""
    KB = K // 128
    ld = ld_for(Mmax)
    As = np.empty((G, Mmax, K), np.uint8)
    sas = np.zeros((G, KB, ld), np.float32)
    for g in range(G):
        As[g], sas[g] = make_a(seed, Mmax, K, stream=STREAM_A + 16 * g, ld_sa=ld)
    B, sb = grouped_b(seed, G, N, K, sigma)
    if masked_m is None:
        masked_m = masked_m_draw(seed, G, Mmax)
    return dict(A=As, sa=sas, ld_sa=ld, B=B, sb=sb, masked_m=np.asarray(masked_m, np.int32),
                G=G, Mmax=Mmax, N=N, K=K)


# The five workloads of the method's benchmark table, by name.
CONFIGS = {
    "dense_128x256x512": dict(kind="dense", M=128, N=256, K=512),
    "dense_64x2112x7168": dict(kind="dense", M=64, N=2112, K=7168),
    "dense_4096x7168x16384": dict(kind="dense", M=4096, N=7168, K=16384, b_sigma=0.02,
                                  outlier_frac=0.01),
    "contiguous_g4_m8192_n4096_k7168": dict(kind="contiguous", G=4, rows_per_group=8192,
                                            N=4096, K=7168),
    "masked_g16_m256_n4096_k7168": dict(kind="masked", G=16, Mmax=256, N=4096, K=7168,
                                        expected_m=128),
}


def config_inputs(name: str, seed: int = 0):
    c = CONFIGS[name]
    if c["kind"] == "dense":
        d = dense_inputs(seed, c["M"], c["N"], c["K"], b_sigma=c.get("b_sigma", 1.0),
                         outlier_frac=c.get("outlier_frac", 0.0))
    elif c["kind"] == "contiguous":
        d = contiguous_inputs(seed, [c["rows_per_group"]] * c["G"], c["N"], c["K"])
    else:
        d = masked_inputs(seed, c["G"], c["Mmax"], c["N"], c["K"])
        d["expected_m"] = c["expected_m"]
    d["kind"] = c["kind"]
    return d
