"""GPU parity of the expert pipeline around the contiguous GEMM
(fp8g_moe_dispatch / fp8g_moe_combine through the C ABI) against the CPU
oracle.  Layout, positions, m_indices, quantised rows, scales and padding are
integer or bit-pattern work and must match bit for bit; the combine fixes its
rounding order (FP32, one fused multiply-add per slot) and must match bit
for bit too.  The end-to-end chain dispatch -> contiguous GEMM -> combine is
compared with the oracle's chain within the GEMM tolerance."""
import numpy as np
import pytest
import torch

import oracle
from fp8_block_scaled_x128_b200 import synth

from .parity_util import bf16_to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from fp8_block_scaled_x128_b200 import gemm
    gemm.device_error(clear=True)
    return gemm


def routing(seed, T, topk, G, drop=0.0, skew=None):
    rng = np.random.default_rng(seed)
    if skew is not None:
        e = np.full(T * topk, skew, np.int32)
    else:
        e = np.stack([rng.choice(G, topk, replace=False) for _ in range(T)]).astype(np.int32).ravel()
    if drop:
        e[rng.random(e.size) < drop] = -1
    return e


def tokens(seed, T, K):
    return synth.round_to_bf16(synth.normal(synth.stream_key(seed, 9), 0, T * K)).reshape(T, K)


def host(t):
    torch.cuda.synchronize()
    return t.cpu().numpy()


def check_dispatch(g, x, e, topk, G, dtype="bf16"):
    T, K = x.shape
    xd = torch.from_numpy(x).cuda()
    if dtype == "bf16":
        xd = xd.to(torch.bfloat16)
    A, sa, pos, mi = g.moe_dispatch(xd, torch.from_numpy(e).cuda(), topk, G)
    blocks = mi.numel()
    used, eA, esa, epos, emi = oracle.moe_dispatch(x, e, topk, G, blocks)
    assert np.array_equal(host(mi), emi)
    assert np.array_equal(host(pos), epos)
    rows = used * 128
    assert np.array_equal(host(A)[:rows], eA[:rows])
    assert np.array_equal(host(sa)[:, :rows], esa[:, :rows])
    return A, sa, pos, mi, used


@pytest.mark.parametrize("T,topk,G,K,drop", [(300, 2, 5, 384, 0.0), (4096, 8, 64, 1024, 0.05), (1, 1, 1, 128, 0.0),
                                             (2500, 6, 256, 256, 0.0), (129, 3, 7, 7168, 0.2),
                                             (200, 12, 16, 256, 0.1)])
def test_dispatch_matches_oracle(g, T, topk, G, K, drop):
    check_dispatch(g, tokens(T + K, T, K), routing(T + G, T, topk, G, drop), topk, G)
    assert g.device_error() == 0


def test_dispatch_skewed_empty_and_float32(g):
    x = tokens(3, 700, 512)
    check_dispatch(g, x, routing(1, 700, 1, 8, skew=5), 1, 8)                  # one hot expert, 7 empty
    check_dispatch(g, x, np.full(700 * 2, -1, np.int32), 2, 4)                # every row dropped
    xf = tokens(4, 300, 256) * np.float32(37.0)
    check_dispatch(g, xf, routing(2, 300, 2, 9), 2, 9, dtype="f32")
    assert g.device_error() == 0


def test_dispatch_flags_bad_expert_ids(g):
    x = tokens(5, 64, 256)
    e = routing(3, 64, 2, 4)
    e[[3, 10]] = [4, -7]                       # out of range: dropped and flagged
    g.device_error(clear=True)
    xd = torch.from_numpy(x).cuda().to(torch.bfloat16)
    A, sa, pos, mi = g.moe_dispatch(xd, torch.from_numpy(e).cuda(), 2, 4)
    p = host(pos)
    assert p[3] == -1 and p[10] == -1
    assert g.device_error() & g.DEVERR_BAD_EXPERT
    e2 = e.copy()
    e2[[3, 10]] = -1
    used, eA, esa, epos, emi = oracle.moe_dispatch(x, e2, 2, 4, mi.numel())
    assert np.array_equal(p, epos) and np.array_equal(host(mi), emi)


@pytest.mark.parametrize("T,topk,N", [(200, 1, 64), (333, 4, 520), (50, 8, 4096), (77, 12, 264)])
def test_combine_matches_oracle_bit_for_bit(g, T, topk, N):
    rng = np.random.default_rng(T + N)
    G = max(6, topk)
    e = routing(T, T, topk, G, drop=0.1)
    used, cnt, off, pos, mi = oracle.moe_layout(e, G, (T * topk + 127) // 128 + G)
    D = synth.bf16_bits(synth.round_to_bf16(rng.standard_normal((max(used, 1) * 128, N)).astype(np.float32)))
    w = rng.uniform(0.0, 1.0, T * topk).astype(np.float32)
    Dd = torch.from_numpy(D.view(np.int16)).cuda().view(torch.bfloat16)
    pd = torch.from_numpy(pos).cuda()
    for wt in (None, w):
        got = g.moe_combine(Dd, pd, None if wt is None else torch.from_numpy(wt).cuda(), T, topk)
        want = oracle.moe_combine(D, pos, wt, T, topk)
        assert np.array_equal(host(got.view(torch.int16)).view(np.uint16), want)


def test_dispatch_gemm_combine_end_to_end(g):
    """Router output -> dispatch -> contiguous GEMM -> combine, against the
    oracle's dispatch, its FP64 contiguous GEMM and an FP64 weighted sum."""
    T, topk, G, N, K = 512, 2, 4, 264, 768
    x = tokens(11, T, K)
    e = routing(12, T, topk, G, drop=0.05)
    w = np.random.default_rng(13).uniform(0.1, 1.0, T * topk).astype(np.float32)
    B, sb = synth.grouped_b(14, G, N, K)
    A, sa, pos, mi = g.moe_dispatch(torch.from_numpy(x).cuda().to(torch.bfloat16), torch.from_numpy(e).cuda(), topk, G)
    M = mi.numel() * 128
    D = g.m_grouped_fp8_gemm_nt_contiguous(A, sa, torch.from_numpy(B).cuda(), torch.from_numpy(sb).cuda(), mi)
    out = g.moe_combine(D, pos, torch.from_numpy(w).cuda(), T, topk)
    got = host(out.view(torch.int16)).view(np.uint16)
    used, eA, esa, epos, emi = oracle.moe_dispatch(x, e, topk, G, mi.numel())
    ex, _ = oracle.m_grouped_contiguous(eA, esa, esa.shape[1], B, sb, emi, M, N, K, G)
    ref, mag, wsum = np.zeros((T, N)), np.zeros((T, N)), np.zeros((T, 1))
    for r in range(T * topk):
        if epos[r] >= 0:
            ref[r // topk] += np.float64(w[r]) * ex[epos[r]]
            mag[r // topk] += np.float64(w[r]) * np.abs(ex[epos[r]])
            wsum[r // topk] += w[r]
    # each D element carries the GEMM tolerance (8e-3 |ex| + 1e-3 rms(ex));
    # the weighted FP32 sum adds nothing measurable; its one bf16 rounding
    # adds at most 2^-9 |ref| (4e-3 with margin)
    rms = float(np.sqrt(np.mean(ex[epos[epos >= 0]] ** 2)))
    err = np.abs(bf16_to_f64(got) - ref)
    lim = 8e-3 * mag + 1e-3 * rms * wsum + 4e-3 * np.abs(ref)
    assert np.all(err <= lim), f"{int(np.sum(err > lim))} elements out of tolerance, worst {np.max(err - lim)}"
    assert g.device_error() == 0
