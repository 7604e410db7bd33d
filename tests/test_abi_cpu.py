"""The C-ABI library on a machine without a GPU: it builds for sm_100a, loads,
exports every entry point declared in include/fp8gemm.h, and rejects bad
arguments on the host before touching the device."""
import ctypes as C
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp8gemm.h")


@pytest.fixture(scope="module")
def lib():
    from fp8_block_scaled_x128_b200 import build
    path = build.build()
    L = C.CDLL(path)
    P, I = C.c_void_p, C.c_int
    L.fp8_gemm_nt.argtypes = [P, P, I, P, P, P, I, I, I, P]
    L.m_grouped_fp8_gemm_nt_contiguous.argtypes = [P, P, I, P, P, P, P, I, I, I, I, P]
    L.m_grouped_fp8_gemm_nt_masked.argtypes = [P, P, I, P, P, P, P, I, I, I, I, I, P]
    L.fp8g_status_string.restype = C.c_char_p
    L.fp8g_variant_name.restype = C.c_char_p
    return L


def declared_functions(path=None):
    """Functions declared by one header, or by every header under include/."""
    import glob
    paths = [path] if path else sorted(glob.glob(os.path.join(ROOT, "include", "*.h")))
    text = "".join(open(p).read() for p in paths)
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(\w+)\s*\(", text, flags=re.M)


def test_header_declares_the_three_entry_points():
    names = declared_functions(HEADER)
    for n in ("fp8_gemm_nt", "m_grouped_fp8_gemm_nt_contiguous", "m_grouped_fp8_gemm_nt_masked"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_library_is_built_for_sm100a():
    from fp8_block_scaled_x128_b200 import build
    assert "arch=compute_100a,code=sm_100a" in " ".join(build.FLAGS)


# fake, never-dereferenced device addresses: every call below returns before any CUDA call
A = B = D = 0x7f0000000000
SA = SB = 0x7f0000100000
S = None


@pytest.mark.parametrize("args,status", [
    ((A, SA, 64, B, SB, D, 64, 2112, 100, S), 1),      # K not a multiple of 128
    ((A, SA, 64, B, SB, D, 64, 2112, 0, S), 1),        # K == 0
    ((A, SA, 64, B, SB, D, 64, 2112, 128 * 513, S), 1),  # K too large
    ((A, SA, 64, B, SB, D, -1, 2112, 128, S), 1),      # negative M
    ((A, SA, 32, B, SB, D, 64, 2112, 128, S), 1),      # ld_sa < M
    ((A, SA, 64, B, SB, D, 64, 2110, 128, S), 2),      # N % 8 != 0
    ((A, SA, 66, B, SB, D, 64, 2112, 128, S), 2),      # ld_sa % 4 != 0
    ((None, SA, 64, B, SB, D, 64, 2112, 128, S), 1),   # null A
    ((A, SA, 64, B, None, D, 64, 2112, 128, S), 1),    # null sb
    ((A + 8, SA, 64, B, SB, D, 64, 2112, 128, S), 2),  # A not 16-byte aligned
    ((A, SA, 64, B, SB, D + 2, 64, 2112, 128, S), 2),  # D not 16-byte aligned
    ((A, SA + 4, 64, B, SB, D, 64, 2112, 128, S), 2),  # sa not 16-byte aligned
    ((A, SA, 64, B, SB + 2, D, 64, 2112, 128, S), 2),  # sb not 4-byte aligned
    ((None, None, 4, None, None, None, 0, 2112, 128, S), 0),  # M == 0: no-op
    ((None, None, 64, None, None, None, 64, 0, 128, S), 0),   # N == 0: no-op
])
def test_dense_host_validation(lib, args, status):
    assert lib.fp8_gemm_nt(*args) == status


def test_contiguous_host_validation(lib):
    f = lib.m_grouped_fp8_gemm_nt_contiguous
    idx = 0x7f0000200000
    assert f(A, SA, 256, B, SB, D, idx, 200, 128, 128, 2, S) == 1       # M % 128 != 0
    assert f(A, SA, 256, B, SB, D, None, 256, 128, 128, 2, S) == 1      # null m_indices
    assert f(A, SA, 256, B, SB, D, idx + 2, 256, 128, 128, 2, S) == 2   # misaligned m_indices
    assert f(A, SA, 256, B, SB, D, idx, 256, 128, 128, -1, S) == 1      # G < 0
    assert f(None, None, 4, None, None, None, None, 0, 128, 128, 2, S) == 0


def test_masked_host_validation(lib):
    f = lib.m_grouped_fp8_gemm_nt_masked
    mm = 0x7f0000200000
    assert f(A, SA, 256, B, SB, D, None, 4, 256, 128, 128, 128, S) == 1   # null masked_m
    assert f(A, SA, 252, B, SB, D, mm, 4, 256, 128, 128, 128, S) == 1     # ld_sa < Mmax
    assert f(A, SA, 256, B, SB, D, mm, 4, 256, 128, 128, -1, S) == 1      # expected_m < 0
    assert f(A, SA, 256, B, SB, D, mm, 4, 256, 130, 128, 128, S) == 2     # N % 8
    assert f(None, None, 256, None, None, None, None, 0, 256, 128, 128, 1, S) == 0  # G == 0


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU error path")
def test_valid_call_without_gpu_reports_cuda_error(lib):
    assert lib.fp8_gemm_nt(A, SA, 64, B, SB, D, 64, 2112, 7168, S) == 4


def test_status_strings_and_variant_table(lib):
    for s in range(6):
        assert lib.fp8g_status_string(s)
    n = lib.fp8g_num_variants()
    assert n >= 3
    names = [lib.fp8g_variant_name(i).decode() for i in range(n)]
    assert len(set(names)) == n
    assert lib.fp8g_variant_name(n) is None
    assert lib.fp8g_set_variant_override(n) == 1
    assert lib.fp8g_set_variant_override(-2) == 1
    assert lib.fp8g_set_variant_override(0) == 0
    assert lib.fp8g_set_variant_override(-1) == 0
    assert lib.fp8g_version() >= 100


def test_every_variant_name_starts_with_its_kind(lib):
    # the GPU parity tests run every variant whose name starts with the
    # call's kind; a variant outside the three prefixes would go untested
    names = [lib.fp8g_variant_name(i).decode() for i in range(lib.fp8g_num_variants())]
    for n in names:
        assert n.split("_", 1)[0] in ("dense", "contiguous", "masked", "bf16", "ue8m0"), n
    for kind in ("dense", "contiguous", "masked", "bf16", "ue8m0"):
        assert any(n.startswith(kind + "_") for n in names), kind


def test_sa_to_mn_major_round_trips_ragged_rows(lib):
    """The host helper turns [G][rows][KB] scales into the library's
    [G][KB][ld_sa] layout: checked against the generator's MN-major output
    for a ragged row count (dense) and a grouped (masked) layout."""
    import numpy as np
    from fp8_block_scaled_x128_b200 import synth
    f = lib.fp8g_sa_to_mn_major
    f.argtypes = [C.c_void_p, C.c_void_p, C.c_int, C.c_int, C.c_int, C.c_int]
    ptr = lambda a: a.ctypes.data_as(C.c_void_p)
    # dense, M = 77 (not a multiple of 4), K = 640
    _, sa = synth.make_a(3, 77, 640)              # [KB][ld_sa], zero beyond row 77
    KB, ld = sa.shape
    rows_major = np.ascontiguousarray(sa[:, :77].T)  # [M][KB], what a row-wise quantiser yields
    out = np.full((KB, ld), np.nan, np.float32)
    assert f(ptr(rows_major), ptr(out), 1, 77, KB, ld) == 0
    assert np.array_equal(out, sa)
    # grouped: [G][Mmax][KB] -> [G][KB][ld_sa]
    d = synth.masked_inputs(4, 3, 37, 8, 384)
    src = np.ascontiguousarray(np.transpose(d["sa"][:, :, :37], (0, 2, 1)))
    out = np.full(d["sa"].shape, np.nan, np.float32)
    assert f(ptr(src), ptr(out), 3, 37, 3, d["ld_sa"]) == 0
    assert np.array_equal(out, d["sa"])
    # argument checks
    assert f(None, ptr(out), 1, 4, 3, 4) == 1
    assert f(ptr(src), ptr(out), 0, 4, 3, 4) == 1       # G < 1
    assert f(ptr(src), ptr(out), 1, 8, 3, 4) == 1       # ld_sa < rows
    assert f(ptr(src), ptr(out), 1, 4, 0, 4) == 1       # KB < 1
    assert f(ptr(src), ptr(out), 1, 5, 3, 6) == 2       # ld_sa % 4 != 0


def test_testing_hook_argument_checks(lib):
    f = lib.fp8g_testing_withhold_stage
    f.argtypes = [C.c_int, C.c_uint]
    assert f(3, 50) == 1            # limit below 100 us
    assert f(3, 2_000_000) == 1     # limit above 1 s
    assert f(3, 2000) == 0
    assert f(-1, 0) == 0            # off again


def test_bf16_host_validation(lib):
    f = lib.bf16_gemm_nt
    f.argtypes = [C.c_void_p, C.c_void_p, C.c_void_p, C.c_int, C.c_int, C.c_int, C.c_void_p]
    assert f(A, B, D, 64, 256, 96, S) == 1          # K % 64 != 0
    assert f(A, B, D, 64, 250, 128, S) == 2         # N % 8 != 0
    assert f(A + 8, B, D, 64, 256, 128, S) == 2     # A not 16-byte aligned
    assert f(None, B, D, 64, 256, 128, S) == 1      # null A
    assert f(None, None, None, 0, 256, 128, S) == 0  # M == 0: no-op


def test_moe_combine_host_validation(lib):
    f = lib.fp8g_moe_combine
    f.argtypes = [C.c_void_p, C.c_int, C.c_void_p, C.c_void_p, C.c_int, C.c_int, C.c_void_p, C.c_void_p]
    assert f(D, 64, A, None, 8, 17, D, S) == 1      # topk above 16
    assert f(D, 64, A, None, 8, 0, D, S) == 1       # topk below 1
    assert f(D, 60, A, None, 8, 4, D, S) == 2       # N % 8 != 0
    assert f(None, 64, A, None, 8, 4, D, S) == 1    # null D
    assert f(None, 64, None, None, 0, 4, None, S) == 0  # T == 0: no-op
