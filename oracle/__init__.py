"""ctypes front-end of the CPU oracle (oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check and by the
benchmark's CPU-baseline leg; never by the library's product path.  It shares
no code with the CUDA path.  Inputs are numpy arrays in the library's boundary
layouts (see oracle.c for the definition and the citations).
"""
from __future__ import annotations

import contextlib
import ctypes as C
import os

import numpy as np

from .build import build

_lib = None


def load(path: str):
    """Load one compiled copy of oracle.c and declare its signatures."""
    L = C.CDLL(path)
    P = C.c_void_p
    i = C.c_int
    L.fp8o_e4m3_value.restype = C.c_double
    L.fp8o_e4m3_value.argtypes = [C.c_uint8]
    L.fp8o_bf16_rne.restype = C.c_uint16
    L.fp8o_bf16_rne.argtypes = [C.c_double]
    L.fp8o_gemm_nt.restype = i
    L.fp8o_gemm_nt.argtypes = [P, P, i, P, P, i, i, i, P, i, P, P, i]
    L.fp8o_m_grouped_contiguous.restype = i
    L.fp8o_m_grouped_contiguous.argtypes = [P, P, i, P, P, P, i, i, i, i, P, i, P, P, i]
    L.fp8o_m_grouped_masked.restype = i
    L.fp8o_m_grouped_masked.argtypes = [P, P, i, P, P, P, i, i, i, i, P, P, i]
    L.fp8o_e4m3_encode.restype = C.c_uint8
    L.fp8o_e4m3_encode.argtypes = [C.c_float]
    L.fp8o_quantize_1x128.restype = i
    L.fp8o_quantize_1x128.argtypes = [P, i, i, P, P, i]
    L.fp8o_quantize_128x128.restype = i
    L.fp8o_quantize_128x128.argtypes = [P, i, i, P, P]
    L.fp8o_moe_layout.restype = i
    L.fp8o_moe_layout.argtypes = [P, i, i, i, P, P, P, P]
    L.fp8o_moe_dispatch.restype = i
    L.fp8o_moe_dispatch.argtypes = [P, i, i, P, i, i, i, P, P, i, P, P]
    L.fp8o_moe_combine.restype = i
    L.fp8o_moe_combine.argtypes = [P, i, P, P, i, i, P]
    L.fp8o_bf16_gemm_nt.restype = i
    L.fp8o_bf16_gemm_nt.argtypes = [P, P, i, i, i, P, i, P, P]
    L.fp8o_ue8m0_value.restype = C.c_double
    L.fp8o_ue8m0_value.argtypes = [C.c_uint8]
    L.fp8o_gemm_nt_ue8m0.restype = i
    L.fp8o_gemm_nt_ue8m0.argtypes = [P, P, i, P, P, i, i, i, P, i, P, P, i]
    return L


@contextlib.contextmanager
def using(path: str):
    """Temporarily route every call to another build of oracle.c (used by the
    mutation tests, which plant mistakes in a copy of the source)."""
    global _lib
    saved = lib()
    _lib = load(path)
    try:
        yield
    finally:
        _lib = saved


def lib():
    global _lib
    if _lib is None:
        _lib = load(build())
    return _lib


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _c(a, dt):
    return np.ascontiguousarray(a, dtype=dt)


def e4m3_value(code: int) -> float:
    return lib().fp8o_e4m3_value(int(code))


def bf16_rne(x: float) -> int:
    return lib().fp8o_bf16_rne(float(x))


def gemm_nt(A, sa, ld_sa, B, sb, M, N, K, rows=None, nthreads=None, out_exact=None, out_bf16=None):
    """Dense NT GEMM.  Returns (exact float64 [nrows, N], bf16 bits uint16 [nrows, N])."""
    A, sa, B, sb = _c(A, np.uint8), _c(sa, np.float32), _c(B, np.uint8), _c(sb, np.float32)
    r = None if rows is None else _c(rows, np.int32)
    nrows = M if r is None else len(r)
    ex = np.zeros((nrows, N), np.float64) if out_exact is None else out_exact
    bf = np.zeros((nrows, N), np.uint16) if out_bf16 is None else out_bf16
    rc = lib().fp8o_gemm_nt(_p(A), _p(sa), int(ld_sa), _p(B), _p(sb), int(M), int(N), int(K),
                            _p(r), int(nrows), _p(ex), _p(bf), int(nthreads or default_threads()))
    if rc:
        raise ValueError("oracle: bad arguments")
    return ex, bf


def m_grouped_contiguous(A, sa, ld_sa, B, sb, m_indices, M, N, K, G, rows=None, nthreads=None,
                         out_exact=None, out_bf16=None):
    """Contiguous grouped GEMM.  Output slots of rows in skipped (-1) blocks keep
    the values passed in (out_exact/out_bf16), default 0."""
    A, sa, B, sb = _c(A, np.uint8), _c(sa, np.float32), _c(B, np.uint8), _c(sb, np.float32)
    mi = _c(m_indices, np.int32)
    r = None if rows is None else _c(rows, np.int32)
    nrows = M if r is None else len(r)
    ex = np.zeros((nrows, N), np.float64) if out_exact is None else out_exact
    bf = np.zeros((nrows, N), np.uint16) if out_bf16 is None else out_bf16
    rc = lib().fp8o_m_grouped_contiguous(_p(A), _p(sa), int(ld_sa), _p(B), _p(sb), _p(mi),
                                         int(M), int(N), int(K), int(G), _p(r), int(nrows),
                                         _p(ex), _p(bf), int(nthreads or default_threads()))
    if rc:
        raise ValueError("oracle: bad arguments")
    return ex, bf


def m_grouped_masked(A, sa, ld_sa, B, sb, masked_m, G, Mmax, N, K, nthreads=None,
                     out_exact=None, out_bf16=None):
    """Masked grouped GEMM over [G, Mmax, N].  Rows m >= masked_m[g] keep the
    values passed in (default 0)."""
    A, sa, B, sb = _c(A, np.uint8), _c(sa, np.float32), _c(B, np.uint8), _c(sb, np.float32)
    mm = _c(masked_m, np.int32)
    ex = np.zeros((G, Mmax, N), np.float64) if out_exact is None else out_exact
    bf = np.zeros((G, Mmax, N), np.uint16) if out_bf16 is None else out_bf16
    rc = lib().fp8o_m_grouped_masked(_p(A), _p(sa), int(ld_sa), _p(B), _p(sb), _p(mm), int(G),
                                     int(Mmax), int(N), int(K), _p(ex), _p(bf),
                                     int(nthreads or default_threads()))
    if rc:
        raise ValueError("oracle: bad arguments")
    return ex, bf


def e4m3_encode(x: float) -> int:
    return lib().fp8o_e4m3_encode(float(x))


def quantize_1x128(x, ld_sa=None):
    """Activations x [rows, K] (float32; bf16 values converted exactly) ->
    (codes uint8 [rows, K], sa float32 [KB, ld_sa]; entries past rows are 0)."""
    x = _c(x, np.float32)
    rows, K = x.shape
    ld = max(4, (rows + 3) // 4 * 4) if ld_sa is None else int(ld_sa)
    q = np.zeros((rows, K), np.uint8)
    sa = np.zeros((K // 128 if K % 128 == 0 else 1, ld), np.float32)
    if lib().fp8o_quantize_1x128(_p(x), int(rows), int(K), _p(q), _p(sa), int(ld)):
        raise ValueError("oracle: bad arguments")
    return q, sa


def quantize_128x128(x):
    """Weights x [N, K] float32 -> (codes uint8 [N, K], sb float32 [NB, KB])."""
    x = _c(x, np.float32)
    N, K = x.shape
    q = np.zeros((N, K), np.uint8)
    sb = np.zeros(((N + 127) // 128, max(1, K // 128)), np.float32)
    if lib().fp8o_quantize_128x128(_p(x), int(N), int(K), _p(q), _p(sb)):
        raise ValueError("oracle: bad arguments")
    return q, sb


def moe_layout(e, G, blocks):
    """Expert layout of routed rows e [R] (int32; -1 = dropped).  Returns
    (blocks_used, cnt [G], off [G], pos [R], m_indices [blocks])."""
    e = _c(e, np.int32)
    R = len(e)
    cnt, off = np.zeros(G, np.int32), np.zeros(G, np.int32)
    pos, mi = np.zeros(R, np.int32), np.zeros(blocks, np.int32)
    used = lib().fp8o_moe_layout(_p(e), R, int(G), int(blocks), _p(cnt), _p(off), _p(pos), _p(mi))
    if used < 0:
        raise ValueError("oracle: bad arguments or too few blocks")
    return used, cnt, off, pos, mi


def moe_dispatch(x, e, topk, G, blocks, ld_sa=None, fill=0):
    """Dispatch with quantisation: x [T, K] float32 token activations, e [T*topk].
    Returns (blocks_used, A [blocks*128, K] uint8, sa [KB, ld_sa], pos, m_indices);
    rows of unused blocks keep `fill`."""
    x = _c(x, np.float32)
    e = _c(e, np.int32)
    T, K = x.shape
    M = blocks * 128
    ld = M if ld_sa is None else int(ld_sa)
    A = np.full((M, K), fill, np.uint8)
    sa = np.zeros((K // 128, ld), np.float32)
    pos, mi = np.zeros(len(e), np.int32), np.zeros(blocks, np.int32)
    used = lib().fp8o_moe_dispatch(_p(x), int(T), int(K), _p(e), int(topk), int(G), int(blocks),
                                   _p(A), _p(sa), int(ld), _p(pos), _p(mi))
    if used < 0:
        raise ValueError("oracle: bad arguments or too few blocks")
    return used, A, sa, pos, mi


def moe_combine(D_bits, pos, w, T, topk):
    """out [T, N] bf16 bits = bf16(sum_k w * D[pos]) in FP32, fused multiply-adds in slot order."""
    D_bits = _c(D_bits, np.uint16)
    pos = _c(pos, np.int32)
    N = D_bits.shape[1]
    wp = None if w is None else _c(w, np.float32)
    out = np.zeros((T, N), np.uint16)
    lib().fp8o_moe_combine(_p(D_bits), int(N), _p(pos), None if wp is None else _p(wp), int(T), int(topk), _p(out))
    return out


def bf16_gemm_nt(A_bits, B_bits, rows=None):
    """BF16 NT GEMM: A [M, K], B [N, K] bf16 bit patterns (uint16).  Returns
    (exact float64 [nrows, N], bf16 bits [nrows, N])."""
    A, B = _c(A_bits, np.uint16), _c(B_bits, np.uint16)
    M, K = A.shape
    N = B.shape[0]
    r = None if rows is None else _c(rows, np.int32)
    nrows = M if r is None else len(r)
    ex = np.zeros((nrows, N), np.float64)
    bf = np.zeros((nrows, N), np.uint16)
    if lib().fp8o_bf16_gemm_nt(_p(A), _p(B), int(M), int(N), int(K), _p(r), int(nrows), _p(ex), _p(bf)):
        raise ValueError("oracle: bad arguments")
    return ex, bf


def ue8m0_value(e: int) -> float:
    return lib().fp8o_ue8m0_value(int(e))


def gemm_nt_ue8m0(A, sfa, ld_sf, B, sfb, M, N, K, rows=None, nthreads=None):
    """Dense NT GEMM with power-of-two scale bytes (UE8M0: 2^(e-127)).
    Returns (exact float64 [nrows, N], bf16 bits [nrows, N])."""
    A, B = _c(A, np.uint8), _c(B, np.uint8)
    sfa, sfb = _c(sfa, np.uint8), _c(sfb, np.uint8)
    r = None if rows is None else _c(rows, np.int32)
    nrows = M if r is None else len(r)
    ex = np.zeros((nrows, N), np.float64)
    bf = np.zeros((nrows, N), np.uint16)
    if lib().fp8o_gemm_nt_ue8m0(_p(A), _p(sfa), int(ld_sf), _p(B), _p(sfb), int(M), int(N), int(K), _p(r),
                                int(nrows), _p(ex), _p(bf), int(nthreads or default_threads())):
        raise ValueError("oracle: bad arguments")
    return ex, bf
