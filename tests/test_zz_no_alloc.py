"""The dense entry point that allocates no device memory, on the GPU.

fp8_gemm_nt_no_alloc is for callers that cannot allocate device memory when
they run a GEMM (a fixed memory pool, or code running during graph capture):
its split-K scratch is a fixed array inside the library instead of a
workspace allocated on first use.  This file is collected last so that a run
stopping at the first failure has already run every other test; it passes
both on its own in a fresh process and after the other tests.
"""
import numpy as np
import pytest
import torch

from fp8_block_scaled_x128_b200 import synth

from .parity_util import assert_close, bf16_to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from fp8_block_scaled_x128_b200 import gemm
    yield gemm
    gemm.set_variant_override(None)


def _dev(d):
    return {k: torch.from_numpy(np.ascontiguousarray(d[k])).cuda() for k in ("A", "sa", "B", "sb")}


def _bits(t):
    torch.cuda.synchronize()
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("shape", [(64, 2112, 7168), (1, 8, 128), (65, 520, 1024)],
                         ids=lambda s: "x".join(map(str, s)))
def test_no_alloc_matches_regular_entry_point_on_two_calls(g, shape):
    M, N, K = shape
    d = synth.dense_inputs(77 + M, M, N, K)
    t = _dev(d)
    ref = _bits(g.fp8_gemm_nt(t["A"], t["sa"], t["B"], t["sb"]))
    D = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    for call in range(2):  # the second call reuses the scratch the first one left behind
        D.view(torch.int16).fill_(0x7F7F)
        g.fp8_gemm_nt_no_alloc(t["A"], t["sa"], t["B"], t["sb"], D=D)
        got = _bits(D)
        assert_close(got, bf16_to_f64(ref), f"no-alloc call {call} {shape}")
    assert g.device_error() == 0


def test_no_alloc_rejects_shapes_beyond_its_scratch(g):
    M, N, K = 256, 8192, 256  # 64 x 4 = 256 tiles > 160 slots
    d = synth.dense_inputs(5, M, N, K)
    t = _dev(d)
    with pytest.raises(g.Fp8GemmError) as e:
        g.fp8_gemm_nt_no_alloc(t["A"], t["sa"], t["B"], t["sb"])
    assert e.value.status == 3
