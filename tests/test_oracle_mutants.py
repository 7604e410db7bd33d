"""Plant one mistake at a time in a copy of the oracle's C source and check
that the pin suite (tests/test_oracle_pins.py) rejects every mutant.

This shows that the pins constrain each part of the definition: the e4m3
decode, the bf16 rounding, both scale indices, the K-block partial, the
operand layout and the grouped-layout bookkeeping.  Only CPU code runs here.
"""
import os
import subprocess

import pytest

import oracle
from oracle.build import SRC as ORACLE_SRC

from . import test_oracle_pins as pins
from . import test_oracle_bf16_pins as bpins
from . import test_oracle_moe_pins as mpins
from . import test_oracle_quant_pins as qpins
from . import test_oracle_ue8m0_pins as upins

MUTANTS = {
    "decode_bias": ("v = ldexp(8.0 + (double)m, e - 7 - 3);", "v = ldexp(8.0 + (double)m, e - 8 - 3);"),
    "decode_sign": ("return s ? -v : v;", "return v;"),
    "decode_subnormal": ("v = ldexp((double)m, -9);", "v = ldexp((double)m, -10);"),
    "bf16_truncates": ("n = nearbyint(a / q);", "n = floor(a / q);"),
    "bf16_ties_away": ("n = nearbyint(a / q);", "n = round(a / q);"),
    "sb_block_index": ("sb[(long)(n / 128) * KB + kb]", "sb[(long)(n / 64) * KB + kb]"),
    "sb_kb_reversed": ("sb[(long)(n / 128) * KB + kb]", "sb[(long)(n / 128) * KB + (KB - 1 - kb)]"),
    "sa_stride_dropped": ("sa_col[(long)kb * sa_stride]", "sa_col[kb]"),
    "sb_dropped": ("acc[n] += (partial * s_a) * s_b;", "acc[n] += (partial * s_a);"),
    "b_kblock_offset": ("B + (long)n * K + (long)kb * 128;", "B + (long)n * K;"),
    "partial_short": ("for (int j = 0; j < 128; ++j)\n                partial", "for (int j = 0; j < 127; ++j)\n                partial"),
    "contig_block_index": ("int g = m_indices[m / 128];", "int g = m_indices[m / 64 < M / 128 ? m / 64 : m / 128];"),
    "contig_no_skip": ("if (g < 0)\n            continue;", "if (g < 0)\n            g = 0;"),
    "masked_row_shift": ("long orow = (long)g * Mmax + m;", "long orow = (long)g * Mmax + (m + 1 < Mmax ? m + 1 : m);"),
    "masked_group_sa": ("sa + (long)g * KB * ld_sa + m", "sa + m"),
    # the FP8 quantiser
    "enc_truncates": ("steps = nearbyint(a / q);", "steps = floor(a / q);"),
    "enc_ties_away": ("steps = nearbyint(a / q);", "steps = round(a / q);"),
    "enc_no_saturation": ("return sign | 0x7E;    /* saturate", "return sign | 0x7F;    /* saturate"),
    "enc_subnormal_quantum": ("if (e < -6)\n        e = -6;", "if (e < -7)\n        e = -7;"),
    "quant_scale_divisor": ("return amax > 0.0f ? amax / 448.0f : 1.0f;", "return amax > 0.0f ? amax / 240.0f : 1.0f;"),
    "quant_group_width": ("for (int j = 0; j < 128; ++j)\n                if (fabsf(g[j]) > amax)",
                          "for (int j = 0; j < 64; ++j)\n                if (fabsf(g[j]) > amax)"),
    "quant_sa_layout": ("sa[(long)kb * ld_sa + r] = s;", "sa[r * KB + kb] = s;"),
    "quant_block_rows": ("for (long r = r0; r < r1; ++r)\n                for (int j = 0; j < 128; ++j) {\n                    float v",
                         "for (long r = r0; r < r0 + 1; ++r)\n                for (int j = 0; j < 128; ++j) {\n                    float v"),
    # the expert pipeline around the contiguous GEMM
    "moe_unstable": ("pos[r] = off[e[r]] + seen[e[r]]++;", "pos[r] = off[e[r]] + (cnt[e[r]] - 1 - seen[e[r]]++);"),
    "moe_extra_block": ("used += (cnt[g] + 127) / 128;", "used += (cnt[g] + 255) / 128;"),
    "moe_m_indices_short": ("b < off[g] / 128 + (cnt[g] + 127) / 128; ++b)", "b < off[g] / 128 + cnt[g] / 128; ++b)"),
    "moe_padding_half_zeroed": ("memset(A + row * K, 0, (size_t)K);", "memset(A + row * K, 0, (size_t)K / 2);"),
    "moe_wrong_token": ("x + (long)(r / topk) * K", "x + (long)(r % topk) * K"),
    "combine_no_weight": ("acc = fmaf(w ? w[r] : 1.0f, d, acc);", "acc = fmaf(1.0f, d, acc);"),
    "combine_unfused": ("acc = fmaf(w ? w[r] : 1.0f, d, acc);", "acc = (w ? w[r] : 1.0f) * d + acc;"),
    # the BF16 GEMM
    "bf16_k_short": ("for (int k = 0; k < K; ++k)\n                acc += arow[k]", "for (int k = 0; k < K - 1; ++k)\n                acc += arow[k]"),
    "bf16_b_transposed": ("bf16_value(B[(long)n * K + k])", "bf16_value(B[(long)k * N + n])"),
    # power-of-two scales
    "ue8m0_bias": ("return e == 255 ? NAN : ldexp(1.0, (int)e - 127);", "return e == 255 ? NAN : ldexp(1.0, (int)e - 126);"),
    "ue8m0_sfb_unused": ("sb[i] = (float)fp8o_ue8m0_value(sfb[i]);", "sb[i] = 1.0f;"),
}

# every pin that takes no parameters, plus the parametrised ones at one or two points
PINS = [
    pins.test_e4m3_decode_all_codes_match_torch,
    pins.test_e4m3_decode_format_landmarks,
    pins.test_bf16_rne_matches_torch_on_float32_values,
    pins.test_bf16_rne_rounds_double_once,
    lambda: [pins.test_worked_examples(c) for c in pins._parse_golden()],
    lambda: pins.test_dense_matches_bruteforce(17, 130, 256),
    lambda: pins.test_dense_matches_bruteforce(33, 257, 256),
    pins.test_dense_ld_sa_padding_and_row_subset,
    pins.test_exact_small_integers_power_of_two_scales,
    pins.test_unit_vector_b_selects_a_column,
    pins.test_doubling_sa_row_doubles_that_row_only,
    pins.test_sb_block_boundary_uses_row_over_128,
    pins.test_contiguous_matches_bruteforce_per_expert_and_skips_minus_one,
    pins.test_contiguous_padding_rows_do_not_affect_other_rows,
    pins.test_masked_rows_beyond_mask_untouched_and_valid_rows_match_bruteforce,
    pins.test_masked_group_permutation_and_independence,
    qpins.test_encode_round_trips_every_finite_code,
    qpins.test_encode_midpoints_round_to_even_and_saturate,
    qpins.test_encode_matches_torch_and_the_generator_on_random_floats,
    lambda: qpins.test_quantize_1x128_against_torch(37, 384),
    qpins.test_quantize_1x128_error_bound_and_locality,
    lambda: qpins.test_quantize_128x128_against_torch(200, 384),
    qpins.test_quantize_128x128_block_is_shared_by_its_rows_only,
    lambda: mpins.test_layout_matches_a_stable_sort(300, 2, 5, 0.0),
    lambda: mpins.test_layout_matches_a_stable_sort(1000, 8, 64, 0.1),
    mpins.test_layout_rejects_too_few_blocks,
    mpins.test_dispatch_rows_are_the_quantised_tokens_and_padding_is_zero,
    mpins.test_combine_is_a_gather_for_one_slot_and_a_weighted_fma_chain,
    mpins.test_combine_rounds_once_per_slot,
    lambda: bpins.test_bf16_gemm_matches_numpy(33, 40, 256),
    bpins.test_bf16_gemm_exact_integers,
    bpins.test_bf16_gemm_closed_forms,
    upins.test_ue8m0_decode,
    upins.test_ue8m0_gemm_matches_bruteforce,
    upins.test_ue8m0_gemm_exact,
]


def _build_mutant(tmp_path, name):
    old, new = MUTANTS[name]
    src = open(ORACLE_SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique"
    path = tmp_path / f"{name}.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / f"lib{name}.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-ffp-contract=off",
                    "-o", str(so), str(path), "-lm"], check=True)
    return str(so)


def test_unmutated_copy_passes_all_pins(tmp_path):
    so = tmp_path / "libclean.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-ffp-contract=off",
                    "-o", str(so), ORACLE_SRC, "-lm"], check=True)
    with oracle.using(str(so)):
        for pin in PINS:
            pin()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_mutant(tmp_path, name):
    so = _build_mutant(tmp_path, name)
    caught = []
    with oracle.using(so):
        for pin in PINS:
            try:
                pin()
            except (AssertionError, ValueError):
                caught.append(getattr(pin, "__name__", "lambda"))
    assert caught, f"mutant {name} survived every pin"
    os.remove(so)
