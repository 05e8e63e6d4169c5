"""The oracle's pins catch plausible mistakes: each case plants one mistake in a copy of the
oracle's C source (on the CPU), compiles it, and runs the pins that guard that function
against it in a subprocess; the pins must fail.  A control compiles the unchanged source the
same way and must pass.

The planted mistakes are the slips a reader of the pages could make: gate and up swapped,
the sign of the SiLU exponent, a scale one power of two too large at exact multiples of 448,
the wrong scale of an all-zero group, a block amax over one row, an off-by-one group count,
the next group's weights, the plain (non-aligned) row order of the prefix-sum layout, a
dropped weight scale, a wrong rounding of E4M3 ties, a wrong scale divisor, row-major
instead of MN-major activation scales, a transposed activation-scale index in the product,
a masked count taken as inclusive, and for the MXFP8 gran-32 recipe a scale index taken per
128 columns, a weight scale read from the wrong row and a block's scale stored at the next
block.
"""
import os
import subprocess
import sys

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = open(os.path.join(ROOT, "oracle", "lnq_oracle.c")).read()

MUTATIONS = {
    "silu_gate_up_swapped": (
        "        h[i] = g[i] / (1.0 + exp(-g[i])) * u[i];",
        "        h[i] = u[i] / (1.0 + exp(-u[i])) * g[i];",
        "tests/test_oracle_silu.py"),
    "silu_exponent_sign": (
        "        h[i] = g[i] / (1.0 + exp(-g[i])) * u[i];",
        "        h[i] = g[i] / (1.0 + exp(g[i])) * u[i];",
        "tests/test_oracle_silu.py"),
    "ue8m0_scale_le": (
        "    while (ldexp(448.0, e) < (double)amax)",
        "    while (ldexp(448.0, e) <= (double)amax)",
        "tests/test_oracle_ue8m0.py"),
    "ue8m0_zero_group": (
        "    if (!(amax > 0.0f))\n        return 0;",
        "    if (!(amax > 0.0f))\n        return -127;",
        "tests/test_oracle_ue8m0.py"),
    "ue8m0_block_one_row": (
        "        e = ue8m0_exponent(amax);\n        sfe[nb * KB + kb]",
        "        e = ue8m0_exponent(fabsf(bf16_bits_to_float(w[n0 * K + kb * ORACLE_GROUP])));\n"
        "        sfe[nb * KB + kb]",
        "tests/test_oracle_ue8m0.py"),
    "psum_count_off_by_one": (
        "        const int64_t c = (int64_t)psum[g] - prev;",
        "        const int64_t c = (int64_t)psum[g] - prev - (g > 0);",
        "tests/test_oracle_psum.py"),
    "psum_next_group_weights": (  # the prefix-sum product's weight row (its indentation is unique)
        "                    dequant_b_row(qb, sfb, K, g * N + n, g * NB + n / ORACLE_GROUP, bd);",
        "                    dequant_b_row(qb, sfb, K, ((g + 1) % G) * N + n, ((g + 1) % G) * NB + n / ORACLE_GROUP, bd);",
        "tests/test_oracle_psum.py"),
    "psum_rows_unaligned": (
        "        start += (c + alignment - 1) / alignment * alignment;",
        "        start += c;",
        "tests/test_oracle_psum.py"),
    "e4m3_ties_away_from_zero": (
        "    f = nearbyint((scaled - 1.0) * 8.0); /* 3-bit mantissa, ties to even */",
        "    f = floor((scaled - 1.0) * 8.0 + 0.5);",
        "tests/test_oracle_e4m3.py"),
    "quantize_scale_divisor": (
        "            s = amax / 448.0f;\n            sfa[g * M4 + m] = s;",
        "            s = amax / 447.0f;\n            sfa[g * M4 + m] = s;",
        "tests/test_oracle_quantize.py"),
    "quantize_scales_row_major": (
        "            sfa[g * M4 + m] = s;",
        "            sfa[m * G + g] = s;",
        "tests/test_oracle_quantize.py"),
    "gemm_activation_scale_index": (
        "(double)sfa[(k / ORACLE_GROUP) * M4 + m];",
        "(double)sfa[(k / ORACLE_GROUP) + m * (K / ORACLE_GROUP)];",
        "tests/test_oracle_gemm.py"),
    "masked_count_inclusive": (
        "            if (m >= masked_m[gr] || !ad || !bd)",
        "            if (m > masked_m[gr] || !ad || !bd)",
        "tests/test_oracle_masked.py"),
    "mx32_product_block_per_128": (
        "            ad[k] = oracle_e4m3_value(qa[m * K + k]) * ldexp(1.0, (int)ea[m * B + k / ORACLE_MX_BLOCK] - 127);",
        "            ad[k] = oracle_e4m3_value(qa[m * K + k]) * ldexp(1.0, (int)ea[m * B + (k / 128) * 4] - 127);",
        "tests/test_oracle_mxfp8.py"),
    "mx32_weight_scale_from_activation_row": (
        "            bd[n * K + k] = oracle_e4m3_value(qb[n * K + k]) * ldexp(1.0, (int)eb[n * B + k / ORACLE_MX_BLOCK] - 127);",
        "            bd[n * K + k] = oracle_e4m3_value(qb[n * K + k]) * ldexp(1.0, (int)eb[k / ORACLE_MX_BLOCK] - 127);",
        "tests/test_oracle_mxfp8.py"),
    "mx32_quantize_scale_of_next_block": (
        "            sfe[r * B + b] = (uint8_t)(e + 127);",
        "            sfe[r * B + (b + 1) % B] = (uint8_t)(e + 127);",
        "tests/test_oracle_mxfp8.py"),
    "gemm_weight_scale_dropped": (
        "        out[k] = oracle_e4m3_value(qb[row * K + k]) * (double)sfb[sb_row * KB + k / ORACLE_GROUP];",
        "        out[k] = oracle_e4m3_value(qb[row * K + k]);",
        "tests/test_oracle_gemm.py"),
}


def run_pins(lib_path: str, test_file: str) -> int:
    env = dict(os.environ, LNQ_ORACLE_LIB=lib_path)
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider", test_file],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return r.returncode


def compile_variant(tmp_path, name: str, text: str) -> str:
    src = tmp_path / f"{name}.c"
    src.write_text(text)
    return oracle.compile_source(str(src), str(tmp_path / f"lib{name}.so"))


def test_control_passes(tmp_path):
    lib = compile_variant(tmp_path, "control", SRC)
    assert run_pins(lib, "tests/test_oracle_ue8m0.py") == 0


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(tmp_path, name):
    old, new, pins = MUTATIONS[name]
    assert SRC.count(old) == 1, f"{name}: the mutated line is not unique in the oracle source"
    lib = compile_variant(tmp_path, name, SRC.replace(old, new))
    assert run_pins(lib, pins) != 0, f"{name}: the pins in {pins} did not catch the planted mistake"
