"""The dense entry point that allocates no device memory, on the GPU.

fp8_gemm_nt_no_alloc serves callers that cannot allocate device memory when
they run a GEMM: an engine that hands out all memory from its own fixed pool,
or a runtime that forbids allocation after start-up.  Its split-K scratch is a
fixed array inside the library instead of a workspace allocated on first use.
The outputs are checked against the CPU oracle (and bit for bit on
exact-integer inputs) on two calls in a row, the second reusing the scratch
the first one left behind.  This file is collected last so that a run
stopping at the first failure has already run every other test; it passes
both on its own in a fresh process and after the other tests.
"""
import numpy as np
import pytest
import torch

import oracle
from fp8_block_scaled_x128_b200 import synth

from .parity_util import assert_close, exact_integer_codes, pow2_scales

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from fp8_block_scaled_x128_b200 import gemm
    gemm.device_error(clear=True)
    yield gemm
    gemm.set_variant_override(None)


def _dev(d):
    return {k: torch.from_numpy(np.ascontiguousarray(d[k])).cuda() for k in ("A", "sa", "B", "sb")}


def _bits(t):
    torch.cuda.synchronize()
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _two_calls(g, d):
    t = _dev(d)
    D = torch.empty((d["M"], d["N"]), dtype=torch.bfloat16, device="cuda")
    out = []
    for _ in range(2):
        D.view(torch.int16).fill_(0x7F7F)
        g.fp8_gemm_nt_no_alloc(t["A"], t["sa"], t["B"], t["sb"], D=D)
        out.append(_bits(D))
    return out


@pytest.mark.parametrize("shape", [(64, 2112, 7168), (1, 8, 128), (65, 520, 1024)],
                         ids=lambda s: "x".join(map(str, s)))
def test_no_alloc_matches_oracle_on_two_calls(g, shape):
    M, N, K = shape
    d = synth.dense_inputs(77 + M, M, N, K)
    ex, _ = oracle.gemm_nt(d["A"], d["sa"], d["ld_sa"], d["B"], d["sb"], M, N, K)
    for call, got in enumerate(_two_calls(g, d)):
        assert_close(got, ex, f"no-alloc call {call} {shape}")
    assert g.device_error() == 0


def test_no_alloc_exact_integers_bit_exact_on_two_calls(g):
    M, N, K = 64, 1040, 2048
    rng = np.random.default_rng(11)
    KB, NB = K // 128, (N + 127) // 128
    ld = synth.ld_for(M)
    sa = np.zeros((KB, ld), np.float32)
    sa[:, :M] = pow2_scales(rng, (KB, M))
    d = dict(A=exact_integer_codes(rng, (M, K)), sa=sa, ld_sa=ld, B=exact_integer_codes(rng, (N, K)),
             sb=pow2_scales(rng, (NB, KB)), M=M, N=N, K=K)
    _, bf = oracle.gemm_nt(d["A"], d["sa"], ld, d["B"], d["sb"], M, N, K)
    for got in _two_calls(g, d):
        assert np.array_equal(got, bf)
    assert g.device_error() == 0


def test_no_alloc_rejects_shapes_beyond_its_scratch(g):
    M, N, K = 256, 8192, 256  # 64 x 4 = 256 tiles > 160 slots
    d = synth.dense_inputs(5, M, N, K)
    t = _dev(d)
    with pytest.raises(g.Fp8GemmError) as e:
        g.fp8_gemm_nt_no_alloc(t["A"], t["sa"], t["B"], t["sb"])
    assert e.value.status == 3
