"""Python binding of the C ABI in include/fp8gemm.h (ctypes; marshalling only).

Every function takes torch CUDA tensors in the library's layouts, passes their
device pointers and the current CUDA stream to libfp8gemm.so, and raises if the
library returns an error.  No step of the GEMM runs in Python or on the CPU; if
the shared library is missing, importing this module raises.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfp8gemm.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m fp8_block_scaled_x128_b200.build` "
        "(the library has no CPU fallback)")

_P, _I, _U32 = C.c_void_p, C.c_int, C.c_uint32

lib = C.CDLL(LIB_PATH)
lib.fp8_gemm_nt.restype = _I
lib.fp8_gemm_nt.argtypes = [_P, _P, _I, _P, _P, _P, _I, _I, _I, _P]
lib.m_grouped_fp8_gemm_nt_contiguous.restype = _I
lib.m_grouped_fp8_gemm_nt_contiguous.argtypes = [_P, _P, _I, _P, _P, _P, _P, _I, _I, _I, _I, _P]
lib.m_grouped_fp8_gemm_nt_masked.restype = _I
lib.m_grouped_fp8_gemm_nt_masked.argtypes = [_P, _P, _I, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P]
lib.fp8_gemm_nt_no_alloc.restype = _I
lib.fp8_gemm_nt_no_alloc.argtypes = [_P, _P, _I, _P, _P, _P, _I, _I, _I, _P]
lib.fp8g_sa_to_mn_major.restype = _I
lib.fp8g_sa_to_mn_major.argtypes = [_P, _P, _I, _I, _I, _I]
lib.fp8g_quantize_1x128.restype = _I
lib.fp8g_quantize_1x128.argtypes = [_P, _I, _I, _I, _P, _P, _I, _P]
lib.fp8g_quantize_128x128.restype = _I
lib.fp8g_quantize_128x128.argtypes = [_P, _I, _I, _I, _P, _P, _P]
lib.fp8g_testing_withhold_stage.restype = _I
lib.fp8g_testing_withhold_stage.argtypes = [_I, C.c_uint]
lib.fp8g_moe_dispatch_workspace_bytes.restype = C.c_size_t
lib.fp8g_moe_dispatch_workspace_bytes.argtypes = [_I, _I]
lib.fp8g_moe_dispatch.restype = _I
lib.fp8g_moe_dispatch.argtypes = [_P, _I, _I, _I, _P, _I, _I, _I, _P, _P, _I, _P, _P, _P, C.c_size_t, _P]
lib.fp8g_moe_combine.restype = _I
lib.fp8g_moe_combine.argtypes = [_P, _I, _P, _P, _I, _I, _P, _P]
lib.bf16_gemm_nt.restype = _I
lib.bf16_gemm_nt.argtypes = [_P, _P, _P, _I, _I, _I, _P]
lib.fp8_gemm_nt_ue8m0.restype = _I
lib.fp8_gemm_nt_ue8m0.argtypes = [_P, _P, _I, _P, _P, _P, _I, _I, _I, _P]
lib.fp8g_status_string.restype = C.c_char_p
lib.fp8g_status_string.argtypes = [_I]
lib.fp8g_get_device_error.restype = _I
lib.fp8g_get_device_error.argtypes = [_I, C.POINTER(_U32), _I]
lib.fp8g_set_variant_override.restype = _I
lib.fp8g_set_variant_override.argtypes = [_I]
lib.fp8g_num_variants.restype = _I
lib.fp8g_num_variants.argtypes = []
lib.fp8g_variant_name.restype = C.c_char_p
lib.fp8g_variant_name.argtypes = [_I]
lib.fp8g_last_variant.restype = _I
lib.fp8g_last_variant.argtypes = []
lib.fp8g_version.restype = _I
lib.fp8g_version.argtypes = []

DEVERR_TIMEOUT, DEVERR_BAD_M_INDEX, DEVERR_MASKED_OVER, DEVERR_BAD_EXPERT = 0x1, 0x2, 0x4, 0x8


class Fp8GemmError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {lib.fp8g_status_string(status).decode()} (status {status})")


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise Fp8GemmError(rc, what)


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream, device):
    s = torch.cuda.current_stream(device) if stream is None else stream
    if s.device != device:
        raise ValueError(f"stream is on {s.device}, the operands on {device}")
    return C.c_void_p(s.cuda_stream)


def _dev(t, dt, name):
    if not t.is_cuda or t.dtype != dt or not t.is_contiguous():
        raise TypeError(f"{name}: expected a contiguous CUDA tensor of {dt}, got {t.dtype} on {t.device}")
    return t


def _one_device(**tensors):
    """The device every operand lives on.  The library encodes its tensor maps
    and launches on the current device, so the call runs under this device and
    operands on different devices are refused before anything is launched."""
    devs = {name: t.device for name, t in tensors.items()}
    first = next(iter(devs.values()))
    for name, d in devs.items():
        if d != first:
            raise ValueError(f"all operands must be on one device: {name} is on {d}, "
                             f"{next(iter(devs))} on {first}")
    return first


def variant_names():
    return [lib.fp8g_variant_name(i).decode() for i in range(lib.fp8g_num_variants())]


def set_variant_override(v: int | None) -> None:
    _check(lib.fp8g_set_variant_override(-1 if v is None else int(v)), "fp8g_set_variant_override")


def testing_withhold_stage(iteration: int | None, wait_limit_us: int = 2000) -> None:
    """Test hook (include/fp8gemm_testing.h): from the next call on, the
    single-CTA kernels skip the loads of pipeline iteration `iteration` and
    give up on any wait after `wait_limit_us`; None turns it off."""
    _check(lib.fp8g_testing_withhold_stage(-1 if iteration is None else int(iteration), int(wait_limit_us)),
           "fp8g_testing_withhold_stage")


def last_variant() -> int:
    return lib.fp8g_last_variant()


def device_error(clear: bool = True, device: int | None = None) -> int:
    """The device error word (FP8G_DEVERR_* bits); synchronises the device."""
    bits = _U32(0)
    d = torch.cuda.current_device() if device is None else device
    rc = lib.fp8g_get_device_error(int(d), C.byref(bits), int(clear))
    if rc not in (0, 5):
        raise Fp8GemmError(rc, "fp8g_get_device_error")
    return bits.value


def fp8_gemm_nt(A, sa, B, sb, D=None, stream=None):
    """Dense: A [M,K] uint8 (e4m3 codes), sa [K/128, ld_sa] float32, B [N,K] uint8,
    sb [ceil(N/128), K/128] float32 -> D [M,N] bfloat16."""
    M, K = A.shape
    N = B.shape[0]
    _dev(A, torch.uint8, "A"), _dev(B, torch.uint8, "B")
    _dev(sa, torch.float32, "sa"), _dev(sb, torch.float32, "sb")
    if D is None:
        D = torch.empty((M, N), dtype=torch.bfloat16, device=A.device)
    _dev(D, torch.bfloat16, "D")
    dev = _one_device(A=A, sa=sa, B=B, sb=sb, D=D)
    with torch.cuda.device(dev):
        _check(lib.fp8_gemm_nt(_ptr(A), _ptr(sa), sa.shape[1], _ptr(B), _ptr(sb), _ptr(D), M, N, K,
                               _stream(stream, dev)), "fp8_gemm_nt")
    return D


def m_grouped_fp8_gemm_nt_contiguous(A, sa, B, sb, m_indices, D=None, stream=None):
    """Contiguous: A [M,K], sa [K/128, ld_sa], B [G,N,K], sb [G, ceil(N/128), K/128],
    m_indices [M/128] int32 -> D [M,N] bfloat16 (rows of -1 blocks untouched)."""
    M, K = A.shape
    G, N, _ = B.shape
    _dev(A, torch.uint8, "A"), _dev(B, torch.uint8, "B"), _dev(m_indices, torch.int32, "m_indices")
    _dev(sa, torch.float32, "sa"), _dev(sb, torch.float32, "sb")
    if D is None:
        D = torch.empty((M, N), dtype=torch.bfloat16, device=A.device)
    _dev(D, torch.bfloat16, "D")
    dev = _one_device(A=A, sa=sa, B=B, sb=sb, D=D, m_indices=m_indices)
    with torch.cuda.device(dev):
        _check(lib.m_grouped_fp8_gemm_nt_contiguous(_ptr(A), _ptr(sa), sa.shape[1], _ptr(B), _ptr(sb), _ptr(D),
                                                    _ptr(m_indices), M, N, K, G, _stream(stream, dev)),
               "m_grouped_fp8_gemm_nt_contiguous")
    return D


def m_grouped_fp8_gemm_nt_masked(A, sa, B, sb, masked_m, expected_m, D=None, stream=None):
    """Masked: A [G,Mmax,K], sa [G, K/128, ld_sa], B [G,N,K], sb [G, ceil(N/128), K/128],
    masked_m [G] int32 (device) -> D [G,Mmax,N] bfloat16 (rows >= masked_m[g] untouched)."""
    G, Mmax, K = A.shape
    N = B.shape[1]
    _dev(A, torch.uint8, "A"), _dev(B, torch.uint8, "B"), _dev(masked_m, torch.int32, "masked_m")
    _dev(sa, torch.float32, "sa"), _dev(sb, torch.float32, "sb")
    if D is None:
        D = torch.empty((G, Mmax, N), dtype=torch.bfloat16, device=A.device)
    _dev(D, torch.bfloat16, "D")
    dev = _one_device(A=A, sa=sa, B=B, sb=sb, D=D, masked_m=masked_m)
    with torch.cuda.device(dev):
        _check(lib.m_grouped_fp8_gemm_nt_masked(_ptr(A), _ptr(sa), sa.shape[2], _ptr(B), _ptr(sb), _ptr(D),
                                                _ptr(masked_m), G, Mmax, N, K, int(expected_m),
                                                _stream(stream, dev)), "m_grouped_fp8_gemm_nt_masked")
    return D


def fp8_gemm_nt_no_alloc(A, sa, B, sb, D=None, stream=None):
    """Dense GEMM like fp8_gemm_nt, for callers that must not allocate device
    memory while they run it (the library keeps this path's split-K scratch in
    a fixed array of its own).  Decode shapes only: at most 160 tiles of 128
    rows of B by 64 rows of A.  Pass D to avoid the output allocation here;
    calls that overlap on the GPU share the scratch and must be ordered."""
    M, K = A.shape
    N = B.shape[0]
    _dev(A, torch.uint8, "A"), _dev(B, torch.uint8, "B")
    _dev(sa, torch.float32, "sa"), _dev(sb, torch.float32, "sb")
    if D is None:
        D = torch.empty((M, N), dtype=torch.bfloat16, device=A.device)
    _dev(D, torch.bfloat16, "D")
    dev = _one_device(A=A, sa=sa, B=B, sb=sb, D=D)
    with torch.cuda.device(dev):
        _check(lib.fp8_gemm_nt_no_alloc(_ptr(A), _ptr(sa), sa.shape[1], _ptr(B), _ptr(sb), _ptr(D), M, N, K,
                                        _stream(stream, dev)), "fp8_gemm_nt_no_alloc")
    return D


def sa_to_mn_major(sa_rows, ld_sa=None):
    """Host helper: A's scales from [rows, KB] (or [G, rows, KB]) float32 to the
    library's MN-major [KB, ld_sa] (or [G, KB, ld_sa]) layout, as a numpy array.
    ld_sa defaults to rows rounded up to a multiple of 4."""
    import numpy as np
    src = np.ascontiguousarray(sa_rows, dtype=np.float32)
    grouped = src.ndim == 3
    if not grouped:
        src = src[None]
    G, rows, KB = src.shape
    ld = max(4, (rows + 3) // 4 * 4) if ld_sa is None else int(ld_sa)
    dst = np.empty((G, KB, ld), np.float32)
    _check(lib.fp8g_sa_to_mn_major(src.ctypes.data_as(_P), dst.ctypes.data_as(_P), G, rows, KB, ld),
           "fp8g_sa_to_mn_major")
    return dst if grouped else dst[0]


_IN_DTYPE = {torch.bfloat16: 0, torch.float32: 1}


def _quant_input(x):
    if not x.is_cuda or x.dtype not in _IN_DTYPE or not x.is_contiguous() or x.dim() != 2:
        raise TypeError(f"x: expected a contiguous 2-D CUDA tensor of bfloat16 or float32, got {x.dtype} "
                        f"{tuple(x.shape)} on {x.device}")
    return x


def quantize_1x128(x, q=None, sa=None, ld_sa=None, stream=None):
    """Activations x [rows, K] (bfloat16 or float32) -> (q [rows, K] uint8 e4m3
    codes, sa [K/128, ld_sa] float32 scales, one per 1x128 group), the GEMM's
    A-side inputs.  ld_sa defaults to rows rounded up to a multiple of 4."""
    _quant_input(x)
    rows, K = x.shape
    ld = max(4, (rows + 3) // 4 * 4) if ld_sa is None else int(ld_sa)
    if q is None:
        q = torch.empty((rows, K), dtype=torch.uint8, device=x.device)
    if sa is None:
        sa = torch.zeros((max(1, K // 128), ld), dtype=torch.float32, device=x.device)
    _dev(q, torch.uint8, "q"), _dev(sa, torch.float32, "sa")
    dev = _one_device(x=x, q=q, sa=sa)
    with torch.cuda.device(dev):
        _check(lib.fp8g_quantize_1x128(_ptr(x), _IN_DTYPE[x.dtype], rows, K, _ptr(q), _ptr(sa), sa.shape[-1],
                                       _stream(stream, dev)), "fp8g_quantize_1x128")
    return q, sa


def quantize_128x128(x, q=None, sb=None, stream=None):
    """Weights x [N, K] (bfloat16 or float32) -> (q [N, K] uint8 e4m3 codes,
    sb [ceil(N/128), K/128] float32 scales, one per 128x128 block)."""
    _quant_input(x)
    N, K = x.shape
    if q is None:
        q = torch.empty((N, K), dtype=torch.uint8, device=x.device)
    if sb is None:
        sb = torch.empty(((N + 127) // 128, max(1, K // 128)), dtype=torch.float32, device=x.device)
    _dev(q, torch.uint8, "q"), _dev(sb, torch.float32, "sb")
    dev = _one_device(x=x, q=q, sb=sb)
    with torch.cuda.device(dev):
        _check(lib.fp8g_quantize_128x128(_ptr(x), _IN_DTYPE[x.dtype], N, K, _ptr(q), _ptr(sb),
                                         _stream(stream, dev)), "fp8g_quantize_128x128")
    return q, sb


def moe_blocks(T: int, topk: int, G: int) -> int:
    """128-row blocks of A that fit any routing of T*topk rows to G experts."""
    return (T * topk + 127) // 128 + G


def moe_dispatch(x, expert, topk, G, blocks=None, out=None, stream=None):
    """Expert dispatch before the contiguous GEMM: x [T, K] (bfloat16 or float32),
    expert [T*topk] int32 (-1 = dropped) -> (A [blocks*128, K] uint8, sa [K/128,
    blocks*128] float32, pos [T*topk] int32, m_indices [blocks] int32).  `out`
    may pass those four tensors (and a workspace as a fifth) to reuse them."""
    _quant_input(x)
    T, K = x.shape
    R = T * topk
    _dev(expert, torch.int32, "expert")
    if expert.numel() != R:
        raise ValueError(f"expert: {expert.numel()} entries for {T} tokens x topk {topk}")
    nb = moe_blocks(T, topk, G) if blocks is None else int(blocks)
    ws_bytes = lib.fp8g_moe_dispatch_workspace_bytes(R, G)
    if ws_bytes == 0:
        raise ValueError(f"moe_dispatch: unsupported R={R}, G={G} (1 <= G <= 256)")
    if out is None:
        A = torch.empty((nb * 128, K), dtype=torch.uint8, device=x.device)
        sa = torch.empty((K // 128, nb * 128), dtype=torch.float32, device=x.device)
        pos = torch.empty(max(R, 1), dtype=torch.int32, device=x.device)
        mi = torch.empty(nb, dtype=torch.int32, device=x.device)
        ws = torch.empty((ws_bytes + 3) // 4, dtype=torch.int32, device=x.device)
    else:
        A, sa, pos, mi, ws = out
    dev = _one_device(x=x, expert=expert, A=A, sa=sa, pos=pos, m_indices=mi, workspace=ws)
    with torch.cuda.device(dev):
        _check(lib.fp8g_moe_dispatch(_ptr(x), _IN_DTYPE[x.dtype], T, K, _ptr(expert), int(topk), int(G), nb,
                                     _ptr(A), _ptr(sa), sa.shape[-1], _ptr(pos), _ptr(mi), _ptr(ws),
                                     ws.numel() * 4, _stream(stream, dev)), "fp8g_moe_dispatch")
    return A, sa, pos[:R], mi


def moe_combine(D, pos, w, T, topk, out=None, stream=None):
    """Combine after the GEMM: out [T, N] bfloat16 = sum over slots of w * D[pos]
    (FP32, one fused multiply-add per slot in slot order); w may be None."""
    _dev(D, torch.bfloat16, "D"), _dev(pos, torch.int32, "pos")
    N = D.shape[-1]
    if w is not None:
        _dev(w, torch.float32, "w")
    if out is None:
        out = torch.empty((T, N), dtype=torch.bfloat16, device=D.device)
    _dev(out, torch.bfloat16, "out")
    tensors = dict(D=D, pos=pos, out=out)
    if w is not None:
        tensors["w"] = w
    dev = _one_device(**tensors)
    with torch.cuda.device(dev):
        _check(lib.fp8g_moe_combine(_ptr(D), N, _ptr(pos), _ptr(w), int(T), int(topk), _ptr(out),
                                    _stream(stream, dev)), "fp8g_moe_combine")
    return out


def bf16_gemm_nt(A, B, D=None, stream=None):
    """BF16 NT GEMM: A [M, K], B [N, K] bfloat16 -> D [M, N] bfloat16 (FP32 accumulation)."""
    _dev(A, torch.bfloat16, "A"), _dev(B, torch.bfloat16, "B")
    M, K = A.shape
    N = B.shape[0]
    if D is None:
        D = torch.empty((M, N), dtype=torch.bfloat16, device=A.device)
    _dev(D, torch.bfloat16, "D")
    dev = _one_device(A=A, B=B, D=D)
    with torch.cuda.device(dev):
        _check(lib.bf16_gemm_nt(_ptr(A), _ptr(B), _ptr(D), M, N, K, _stream(stream, dev)), "bf16_gemm_nt")
    return D


def fp8_gemm_nt_ue8m0(A, sfa, B, sfb, D=None, stream=None):
    """Dense NT GEMM with power-of-two scales: A [M,K] uint8 e4m3, sfa [K/128, ld]
    uint8 (E8M0: 2^(e-127)), B [N,K] uint8, sfb [ceil(N/128), K/128] uint8 ->
    D [M,N] bfloat16 (block-scaled tensor-core MMA, FP32 accumulation over K)."""
    M, K = A.shape
    N = B.shape[0]
    _dev(A, torch.uint8, "A"), _dev(B, torch.uint8, "B"), _dev(sfa, torch.uint8, "sfa"), _dev(sfb, torch.uint8, "sfb")
    if D is None:
        D = torch.empty((M, N), dtype=torch.bfloat16, device=A.device)
    _dev(D, torch.bfloat16, "D")
    dev = _one_device(A=A, sfa=sfa, B=B, sfb=sfb, D=D)
    with torch.cuda.device(dev):
        _check(lib.fp8_gemm_nt_ue8m0(_ptr(A), _ptr(sfa), sfa.shape[1], _ptr(B), _ptr(sfb), _ptr(D), M, N, K,
                                     _stream(stream, dev)), "fp8_gemm_nt_ue8m0")
    return D
