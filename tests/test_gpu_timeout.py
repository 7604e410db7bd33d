"""The device timeout path, exercised on a healthy GPU without a fault.

Every pipeline wait in the kernels is bounded.  The test hook of
include/fp8gemm_testing.h makes the TMA producers of the single-CTA kernel
skip the loads of one pipeline iteration and shortens the wait limit to 2 ms:
nothing is ever in flight on the withheld stage, so the MMA issuer's wait for
it runs out, the kernel records FP8G_DEVERR_TIMEOUT, drains what it has in
flight, frees its tensor memory and returns.  The next normal call on the
same GPU must then be correct again."""
import numpy as np
import pytest
import torch

import oracle
from fp8_block_scaled_x128_b200 import synth

from .parity_util import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from fp8_block_scaled_x128_b200 import gemm
    gemm.device_error(clear=True)
    yield gemm
    gemm.testing_withhold_stage(None)
    gemm.set_variant_override(None)


def _run(g, d, variant):
    t = {k: torch.from_numpy(np.ascontiguousarray(d[k])).cuda() for k in ("A", "sa", "B", "sb")}
    g.set_variant_override(variant)
    try:
        D = g.fp8_gemm_nt(t["A"], t["sa"], t["B"], t["sb"])
        torch.cuda.synchronize()   # raises if the kernel faulted; it must not
        return D.view(torch.int16).cpu().numpy().view(np.uint16)
    finally:
        g.set_variant_override(None)


@pytest.mark.parametrize("vname", ["dense_mlanes_bn128_st6", "dense_nlanes_bn64_st8"])
def test_withheld_stage_times_out_and_the_gpu_stays_usable(g, vname):
    v = g.variant_names().index(vname)
    d = synth.dense_inputs(5, 256, 512, 1024)            # 8 K-blocks per tile
    g.device_error(clear=True)
    g.testing_withhold_stage(3, wait_limit_us=2000)
    try:
        _run(g, d, v)
    finally:
        g.testing_withhold_stage(None)
    bits = g.device_error(clear=True)
    assert bits & g.DEVERR_TIMEOUT, f"expected the timeout bit, got {bits:#x}"
    # the same GPU, the same variant, no hook: correct again, and no error
    ex, _ = oracle.gemm_nt(d["A"], d["sa"], d["ld_sa"], d["B"], d["sb"], d["M"], d["N"], d["K"])
    assert_close(_run(g, d, v), ex, f"{vname} after a timeout")
    assert g.device_error() == 0
