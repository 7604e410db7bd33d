"""The Python binding's argument checks, on a machine without a GPU.

The library encodes its tensor maps and launches on the current CUDA device,
so the binding must refuse operands that live on different devices before it
calls into the library.  Stand-in tensor objects carry only the metadata the
checks read; nothing here touches a device."""
import numpy as np
import pytest
import torch


class FakeCudaTensor:
    def __init__(self, shape, dtype, index):
        self.shape = tuple(shape)
        self.dtype = dtype
        self.device = torch.device("cuda", index)
        self.is_cuda = True

    def is_contiguous(self):
        return True

    def data_ptr(self):
        raise AssertionError("the binding reached the library with operands on two devices")


@pytest.fixture(scope="module")
def gemm():
    from fp8_block_scaled_x128_b200 import gemm
    return gemm


def dense_operands(dev_of):
    M, N, K = 64, 256, 512
    return dict(A=FakeCudaTensor((M, K), torch.uint8, dev_of("A")),
                sa=FakeCudaTensor((K // 128, M), torch.float32, dev_of("sa")),
                B=FakeCudaTensor((N, K), torch.uint8, dev_of("B")),
                sb=FakeCudaTensor((N // 128, K // 128), torch.float32, dev_of("sb")),
                D=FakeCudaTensor((M, N), torch.bfloat16, dev_of("D")))


@pytest.mark.parametrize("odd", ["sa", "B", "sb", "D"])
def test_dense_refuses_operands_on_two_devices(gemm, odd):
    t = dense_operands(lambda name: 1 if name == odd else 0)
    with pytest.raises(ValueError, match="one device"):
        gemm.fp8_gemm_nt(t["A"], t["sa"], t["B"], t["sb"], D=t["D"])
    with pytest.raises(ValueError, match="one device"):
        gemm.fp8_gemm_nt_no_alloc(t["A"], t["sa"], t["B"], t["sb"], D=t["D"])


def test_grouped_calls_refuse_index_tensor_on_another_device(gemm):
    G, M, N, K = 2, 256, 256, 512
    A = FakeCudaTensor((M, K), torch.uint8, 0)
    sa = FakeCudaTensor((K // 128, M), torch.float32, 0)
    B = FakeCudaTensor((G, N, K), torch.uint8, 0)
    sb = FakeCudaTensor((G, N // 128, K // 128), torch.float32, 0)
    D = FakeCudaTensor((M, N), torch.bfloat16, 0)
    idx = FakeCudaTensor((M // 128,), torch.int32, 3)
    with pytest.raises(ValueError, match="m_indices"):
        gemm.m_grouped_fp8_gemm_nt_contiguous(A, sa, B, sb, idx, D=D)
    Am = FakeCudaTensor((G, 128, K), torch.uint8, 0)
    sam = FakeCudaTensor((G, K // 128, 128), torch.float32, 0)
    Dm = FakeCudaTensor((G, 128, N), torch.bfloat16, 0)
    mm = FakeCudaTensor((G,), torch.int32, 2)
    with pytest.raises(ValueError, match="masked_m"):
        gemm.m_grouped_fp8_gemm_nt_masked(Am, sam, B, sb, mm, 64, D=Dm)


def test_wrong_dtype_is_refused(gemm):
    t = dense_operands(lambda name: 0)
    t["sb"].dtype = torch.float16
    with pytest.raises(TypeError, match="sb"):
        gemm.fp8_gemm_nt(t["A"], t["sa"], t["B"], t["sb"], D=t["D"])


def test_sa_to_mn_major_binding(gemm):
    rng = np.random.default_rng(0)
    src = rng.standard_normal((5, 3)).astype(np.float32)   # [rows=5, KB=3]
    out = gemm.sa_to_mn_major(src)
    assert out.shape == (3, 8)
    assert np.array_equal(out[:, :5], src.T) and np.all(out[:, 5:] == 0)
    grp = rng.standard_normal((2, 5, 3)).astype(np.float32)
    out = gemm.sa_to_mn_major(grp, ld_sa=12)
    assert out.shape == (2, 3, 12)
    assert np.array_equal(out[1, :, :5], grp[1].T)
    with pytest.raises(gemm.Fp8GemmError):
        gemm.sa_to_mn_major(src, ld_sa=6)
