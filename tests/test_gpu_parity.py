"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Inputs come from the seeded generator; expected values come from the oracle
only.  Floating-point cases use the acceptance tolerance of parity_util;
exact-integer cases (codes in {-2..2}, power-of-two scales) must match the
oracle's bf16 bits exactly.  Rows that the method must not write (masked rows
past masked_m, contiguous blocks marked -1) are checked bit-for-bit against
a canary fill.
"""
import numpy as np
import pytest
import torch

import oracle
from fp8_block_scaled_x128_b200 import synth

from .parity_util import CANARY, assert_close, exact_integer_codes, pow2_scales

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from fp8_block_scaled_x128_b200 import gemm
    gemm.device_error(clear=True)
    yield gemm
    gemm.set_variant_override(None)


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host_bits(t):
    torch.cuda.synchronize()
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def canary_like(shape):
    return torch.full(shape, CANARY - 0x10000, dtype=torch.int16, device="cuda").view(torch.bfloat16)


def variants(g, prefix):
    return [i for i, n in enumerate(g.variant_names()) if n.startswith(prefix)]


def dense_gpu(g, d, variant=None):
    g.set_variant_override(variant)
    try:
        D = g.fp8_gemm_nt(dev(d["A"]), dev(d["sa"]), dev(d["B"]), dev(d["sb"]))
        if variant is not None:
            assert g.last_variant() == variant
        return host_bits(D)
    finally:
        g.set_variant_override(None)


def exact_dense(seed, M, N, K):
    rng = np.random.default_rng(seed)
    KB, NB = K // 128, (N + 127) // 128
    ld = synth.ld_for(M)
    sa = np.zeros((KB, ld), np.float32)
    sa[:, :M] = pow2_scales(rng, (KB, M))
    return dict(A=exact_integer_codes(rng, (M, K)), sa=sa, ld_sa=ld, B=exact_integer_codes(rng, (N, K)),
                sb=pow2_scales(rng, (NB, KB)), M=M, N=N, K=K)


def oracle_dense(d, rows=None):
    return oracle.gemm_nt(d["A"], d["sa"], d["ld_sa"], d["B"], d["sb"], d["M"], d["N"], d["K"], rows=rows)


# --------------------------------------------------------------------------- dense

DENSE_SHAPES = [(1, 8, 128), (64, 256, 384), (65, 200, 256), (128, 256, 512), (200, 136, 1024),
                (257, 520, 256), (64, 2112, 2048)]


@pytest.mark.parametrize("shape", DENSE_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_dense_every_variant(g, shape):
    M, N, K = shape
    d = synth.dense_inputs(100 + M + N, M, N, K)
    ex, _ = oracle_dense(d)
    for v in variants(g, "dense_"):
        assert_close(dense_gpu(g, d, v), ex, f"{g.variant_names()[v]} {shape}")
    assert g.device_error() == 0


@pytest.mark.parametrize("shape", [(64, 256, 1024), (130, 264, 512), (64, 2112, 7168)],
                         ids=lambda s: "x".join(map(str, s)))
def test_dense_exact_integers_bit_exact(g, shape):
    d = exact_dense(7, *shape)
    _, bf = oracle_dense(d)
    for v in variants(g, "dense_"):
        got = dense_gpu(g, d, v)
        assert np.array_equal(got, bf), g.variant_names()[v]


def test_dense_config_128x256x512(g):
    d = synth.config_inputs("dense_128x256x512")
    ex, _ = oracle_dense(d)
    assert_close(dense_gpu(g, d), ex, "dense_128x256x512")


def test_dense_config_64x2112x7168_all_variants(g):
    d = synth.config_inputs("dense_64x2112x7168")
    ex, _ = oracle_dense(d)
    assert_close(dense_gpu(g, d), ex, "auto")
    for v in variants(g, "dense_"):
        assert_close(dense_gpu(g, d, v), ex, g.variant_names()[v])


@pytest.mark.parametrize("shape", [(1, 8, 128), (65, 200, 256), (257, 520, 256), (64, 2112, 7168)],
                         ids=lambda s: "x".join(map(str, s)))
def test_dense_after_quantiser_in_one_graph(g, shape):
    """Quantiser then GEMM, both programmatic dependent launches (the GEMM's
    prologue may run while the quantiser finishes): in one graph the 1x128
    quantiser writes A and sa right before each GEMM, alternating between two
    activations, and every GEMM must use the A written just before it.  Each
    kernel variant's graph output equals, bit for bit, the same two steps run
    one call at a time; the quantise-then-GEMM result matches the oracles."""
    M, N, K = shape
    d = exact_dense(11, M, N, K)
    B, sb = dev(d["B"]), dev(d["sb"])
    gen = torch.Generator(device="cuda").manual_seed(M + N + K)
    xs = [torch.randn(M, K, device="cuda", generator=gen).to(torch.bfloat16) for _ in range(2)]
    ld = synth.ld_for(M)
    A = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    sa = torch.zeros((K // 128, ld), dtype=torch.float32, device="cuda")
    q0, sa0 = oracle.quantize_1x128(xs[0].float().cpu().numpy(), ld_sa=ld)
    ex, _ = oracle.gemm_nt(q0, sa0, ld, d["B"], d["sb"], M, N, K)
    for v in variants(g, "dense_"):
        g.set_variant_override(v)
        try:
            refs = []
            for x in xs:
                g.quantize_1x128(x, q=A, sa=sa, ld_sa=ld)
                refs.append(host_bits(g.fp8_gemm_nt(A, sa, B, sb)))
            assert_close(refs[0], ex, f"{g.variant_names()[v]} {shape}")
            outs = [canary_like((M, N)) for _ in range(4)]
            stream = torch.cuda.Stream()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=stream):
                for i in range(4):
                    g.quantize_1x128(xs[i % 2], q=A, sa=sa, ld_sa=ld, stream=stream)
                    g.fp8_gemm_nt(A, sa, B, sb, D=outs[i], stream=stream)
            graph.replay()
            torch.cuda.synchronize()
            for i in range(4):
                assert np.array_equal(host_bits(outs[i]), refs[i % 2]), (g.variant_names()[v], i)
            del graph
        finally:
            g.set_variant_override(None)
    assert g.device_error() == 0


def test_dense_is_deterministic(g):
    d = synth.config_inputs("dense_64x2112x7168")
    first = dense_gpu(g, d)
    for _ in range(3):
        assert np.array_equal(dense_gpu(g, d), first)


# --------------------------------------------------------------------------- contiguous

def contig_gpu(g, d, variant=None):
    g.set_variant_override(variant)
    try:
        D = canary_like((d["M"], d["N"]))
        g.m_grouped_fp8_gemm_nt_contiguous(dev(d["A"]), dev(d["sa"]), dev(d["B"]), dev(d["sb"]),
                                           dev(d["m_indices"]), D=D)
        if variant is not None:
            assert g.last_variant() == variant
        return host_bits(D)
    finally:
        g.set_variant_override(None)


def check_contig(g, d, exact=False):
    M, N = d["M"], d["N"]
    ex, bf = oracle.m_grouped_contiguous(d["A"], d["sa"], d["ld_sa"], d["B"], d["sb"], d["m_indices"],
                                         M, N, d["K"], d["G"])
    live = np.repeat(d["m_indices"] >= 0, 128)
    for v in variants(g, "contiguous_"):
        got = contig_gpu(g, d, v)
        name = g.variant_names()[v]
        assert np.all(got[~live] == CANARY), f"{name}: skipped block written"
        if exact:
            assert np.array_equal(got[live], bf[live]), name
        else:
            assert_close(got[live], ex[live], name)


def test_contiguous_ragged_experts_and_skipped_blocks(g):
    d = synth.contiguous_inputs(21, [100, 256, 20, 300], 136, 512, empty_blocks=(1, 5))
    check_contig(g, d)
    assert g.device_error() == 0


def test_contiguous_exact_integers(g):
    d = synth.contiguous_inputs(22, [128, 200, 64], 264, 384, empty_blocks=(2,))
    rng = np.random.default_rng(5)
    d["A"] = exact_integer_codes(rng, d["A"].shape)
    d["B"] = exact_integer_codes(rng, d["B"].shape)
    d["sa"][:, :d["M"]] = pow2_scales(rng, (d["K"] // 128, d["M"]))
    d["sb"] = pow2_scales(rng, d["sb"].shape)
    check_contig(g, d, exact=True)


def test_contiguous_bad_expert_index_is_flagged_and_skipped(g):
    d = synth.contiguous_inputs(23, [128, 128], 64, 128)
    d["m_indices"] = np.array([0, 7], np.int32)  # 7 >= G
    g.device_error(clear=True)
    got = contig_gpu(g, d)
    assert np.all(got[128:] == CANARY)
    assert g.device_error() & g.DEVERR_BAD_M_INDEX


# --------------------------------------------------------------------------- masked

def masked_gpu(g, d, variant=None, expected_m=None):
    g.set_variant_override(variant)
    try:
        D = canary_like((d["G"], d["Mmax"], d["N"]))
        g.m_grouped_fp8_gemm_nt_masked(dev(d["A"]), dev(d["sa"]), dev(d["B"]), dev(d["sb"]),
                                       dev(d["masked_m"]), d["Mmax"] // 2 if expected_m is None else expected_m,
                                       D=D)
        if variant is not None:
            assert g.last_variant() == variant
        return host_bits(D)
    finally:
        g.set_variant_override(None)


def check_masked(g, d, exact=False):
    G, Mmax, N, K = d["G"], d["Mmax"], d["N"], d["K"]
    ex, bf = oracle.m_grouped_masked(d["A"], d["sa"], d["ld_sa"], d["B"], d["sb"], d["masked_m"], G, Mmax, N, K)
    mm = np.minimum(d["masked_m"], Mmax)
    live = np.arange(Mmax)[None, :] < mm[:, None]
    for v in variants(g, "masked_"):
        got = masked_gpu(g, d, v)
        name = g.variant_names()[v]
        assert np.all(got[~live] == CANARY), f"{name}: masked row written"
        if exact:
            assert np.array_equal(got[live], bf[live]), name
        else:
            assert_close(got[live], ex[live], name)


@pytest.mark.parametrize("Mmax,mm", [(40, [0, 1, 39, 40]), (130, [129, 64, 0, 1, 130, 65]),
                                     (256, [255, 256, 0, 1, 127, 128, 129])])
def test_masked_edge_counts(g, Mmax, mm):
    d = synth.masked_inputs(30 + Mmax, len(mm), Mmax, 136, 256, masked_m=mm)
    check_masked(g, d)
    assert g.device_error() == 0


def test_masked_exact_integers(g):
    G, Mmax, N, K = 3, 160, 264, 384
    d = synth.masked_inputs(31, G, Mmax, N, K, masked_m=[160, 33, 97])
    rng = np.random.default_rng(6)
    d["A"] = exact_integer_codes(rng, d["A"].shape)
    d["B"] = exact_integer_codes(rng, d["B"].shape)
    d["sa"][:, :, :Mmax] = pow2_scales(rng, (G, K // 128, Mmax))
    d["sb"] = pow2_scales(rng, d["sb"].shape)
    check_masked(g, d, exact=True)


def test_masked_count_above_mmax_is_clamped_and_flagged(g):
    d = synth.masked_inputs(32, 2, 64, 64, 128, masked_m=[64, 64])
    ref = masked_gpu(g, d)
    d["masked_m"] = np.array([1000, 64], np.int32)
    g.device_error(clear=True)
    got = masked_gpu(g, d)
    assert np.array_equal(got, ref)
    assert g.device_error() & g.DEVERR_MASKED_OVER


def test_masked_expected_m_does_not_change_results(g):
    d = synth.masked_inputs(33, 4, 128, 264, 256, masked_m=[5, 128, 70, 0])
    a = masked_gpu(g, d, expected_m=1)
    b = masked_gpu(g, d, expected_m=128)
    assert np.array_equal(a, b)


def test_masked_in_cuda_graph_reads_counts_on_device(g):
    """The host never reads masked_m: a captured graph replays with new counts."""
    d = synth.masked_inputs(34, 4, 128, 136, 256, masked_m=[128, 128, 128, 128])
    A, sa, B, sb = dev(d["A"]), dev(d["sa"]), dev(d["B"]), dev(d["sb"])
    mm = dev(np.array([128, 128, 128, 128], np.int32))
    D = canary_like((4, 128, 136))
    g.m_grouped_fp8_gemm_nt_masked(A, sa, B, sb, mm, 64, D=D)  # warm-up (per-device set-up)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        g.m_grouped_fp8_gemm_nt_masked(A, sa, B, sb, mm, 64, D=D)
    new = np.array([3, 0, 100, 128], np.int32)
    mm.copy_(torch.from_numpy(new))
    D.view(torch.int16).fill_(CANARY - 0x10000)
    graph.replay()
    got = host_bits(D)
    d["masked_m"] = new
    ex, _ = oracle.m_grouped_masked(d["A"], d["sa"], d["ld_sa"], d["B"], d["sb"], new, 4, 128, 136, 256)
    live = np.arange(128)[None, :] < new[:, None]
    assert np.all(got[~live] == CANARY)
    assert_close(got[live], ex[live], "graph replay")


# --------------------------------------------------------------------------- full-size configurations

def outlier_rows(seed, M, K, frac):
    """Rows of A holding at least one x50 group, read from the generator's own
    outlier stream (the same draw make_a uses), not from the oracle."""
    KB = K // 128
    u = synth.uniform(synth.stream_key(seed, synth.STREAM_OUTLIER), 0, M * KB).reshape(M, KB)
    return np.nonzero((u < frac).any(axis=1))[0].astype(np.int32)


@pytest.mark.slow
def test_config_dense_4096x7168x16384_sampled_rows(g):
    name = "dense_4096x7168x16384"
    d = synth.config_inputs(name)
    got = dense_gpu(g, d)
    rng = np.random.default_rng(0)
    # a random row subsample, compared on all N columns
    rows = np.unique(np.r_[0, 4095, 127, 128, rng.choice(4096, 44, replace=False)]).astype(np.int32)
    ex, _ = oracle_dense(d, rows=rows)
    assert_close(got[rows], ex, f"{name} sampled rows")
    # every row that holds a x50 group, on one 128-column block of B (the
    # oracle computes those columns from that block's rows of B and sb)
    orows = outlier_rows(0, d["M"], d["K"], synth.CONFIGS[name]["outlier_frac"])
    assert 0.6 * d["M"] < len(orows) < 0.85 * d["M"]  # 1 - 0.99^128 of the rows
    for nb in (int(rng.integers(0, d["N"] // 128)), d["N"] // 128 - 1):
        cols = slice(128 * nb, 128 * nb + 128)
        ex, _ = oracle.gemm_nt(d["A"], d["sa"], d["ld_sa"], d["B"][cols], d["sb"][nb:nb + 1], d["M"], 128,
                               d["K"], rows=orows)
        assert_close(got[orows, cols], ex, f"{name} outlier rows, columns {cols}")


@pytest.mark.slow
def test_config_contiguous_sampled_rows(g):
    d = synth.config_inputs("contiguous_g4_m8192_n4096_k7168")
    D = canary_like((d["M"], d["N"]))
    g.m_grouped_fp8_gemm_nt_contiguous(dev(d["A"]), dev(d["sa"]), dev(d["B"]), dev(d["sb"]),
                                       dev(d["m_indices"]), D=D)
    got = host_bits(D)
    rng = np.random.default_rng(1)
    rows = np.unique(np.r_[[8192 * e + o for e in range(4) for o in (0, 8191)],
                           rng.choice(d["M"], 56, replace=False)]).astype(np.int32)
    ex, _ = oracle.m_grouped_contiguous(d["A"], d["sa"], d["ld_sa"], d["B"], d["sb"], d["m_indices"], d["M"],
                                        d["N"], d["K"], d["G"], rows=rows)
    assert_close(got[rows], ex, "contiguous sampled")


@pytest.mark.slow
def test_config_masked_in_full(g):
    d = synth.config_inputs("masked_g16_m256_n4096_k7168")
    got = masked_gpu(g, d, expected_m=d["expected_m"])
    G, Mmax, N, K = d["G"], d["Mmax"], d["N"], d["K"]
    mm = np.minimum(d["masked_m"], Mmax)
    live = np.arange(Mmax)[None, :] < mm[:, None]
    assert np.all(got[~live] == CANARY)
    ex, _ = oracle.m_grouped_masked(d["A"], d["sa"], d["ld_sa"], d["B"], d["sb"], d["masked_m"], G, Mmax, N, K)
    for gi in range(G):
        assert_close(got[gi][:mm[gi]], ex[gi][:mm[gi]], f"masked group {gi} ({mm[gi]} rows)")
    assert g.device_error() == 0
