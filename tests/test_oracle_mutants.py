"""The pins must reject plausible mistakes in the oracle.

Each case copies ``oracle/w4a16_oracle.c``, plants one mistake on the CPU (a
reversed nibble order, a dropped bias, a transposed index, FP64 accumulation,
fused multiply-adds, truncating output rounding, ...), builds the copy with the
same flags and runs every pin against it in a child process.  At least one pin
has to fail for each mutant; the real source must pass them all.
"""
import os
import subprocess
import sys

import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))

MUTANTS = {
    "nibble_order_reversed": ("(word >> (4 * (k % 8)))", "(word >> (4 * (7 - k % 8)))"),
    "code_mask_3_bits": ("& 15u);", "& 7u);"),
    "word_index_stride": ("wq[n * (K / 8) + k / 8]", "wq[n * (K / 16) + k / 8]"),
    "bias_dropped": ("const float w = sq + bi;", "const float w = sq;"),
    "bias_sign": ("const float w = sq + bi;", "const float w = sq - bi;"),
    "scale_dropped": ("const float sq = sc * q;", "const float sq = q;"),
    "scale_group_index": ("bf16_to_f32(s[n * G + k / 128])", "bf16_to_f32(s[n * G + (k / 128) % 1])"),
    "bias_from_scales": ("bf16_to_f32(b[n * G + k / 128])", "bf16_to_f32(s[n * G + k / 128])"),
    "x_row_from_n": ("x[m * K + k]", "x[(n % 1 + m) * K + (k ^ 1)]"),
    "fp64_accumulator": ("float acc = 0.0f;", "double acc = 0.0;"),
    "truncating_round": ("u += 0x7fffu + ((u >> 16) & 1u);", "u += 0u;"),
    "ties_away": ("u += 0x7fffu + ((u >> 16) & 1u);", "u += 0x8000u;"),
    "k_descending": ("for (int64_t k = 0; k < K; ++k) {", "for (int64_t k = K - 1; k >= 0; --k) {"),
    # quantiser
    "quant_truncates": ("const float r = nearbyintf(t);", "const float r = truncf(t);"),
    "quant_ties_away": ("const float r = nearbyintf(t);", "const float r = roundf(t);"),
    "quant_step_16": ("const float step = range / 15.0f;", "const float step = range / 16.0f;"),
    "quant_bias_unrounded": ("const float bi = bf16_to_f32(*bias);", "const float bi = lo;"),
    "quant_no_upper_clamp": ("(r > 15.0f ? 15u : (uint32_t)r)", "((uint32_t)r & 0xFu)"),
    "quant_min_as_max": ("if (v[j] < lo)", "if (v[j] > lo)"),
    "quant_zero_sign_kept": ("    if (lo == 0.0f)\n        lo = 0.0f;\n", ""),
    "quant_words_not_cleared": ("        words[j] = 0u;", "        words[j] = 1u;"),
    "quant_nibble_order": ("code << (4 * (j % 8))", "code << (4 * (7 - j % 8))"),
    # fused gate/up
    "gate_rows_not_interleaved": ("gate_row = 16 * (j / 8) + j % 8;", "gate_row = 8 * (j / 8) + j % 8;"),
    "up_row_is_gate_row": ("const int64_t up_row = gate_row + 8;", "const int64_t up_row = gate_row;"),
    "silu_sign": ("return g / (1.0 + exp(-g));", "return g / (1.0 + exp(g));"),
    "silu_dropped": ("f32_to_bf16_rne((float)(silu(gv) * uv))", "f32_to_bf16_rne((float)(gv * uv))"),
    # other bit widths
    "bits_code_order_reversed": ("(word >> (bits * (k % per_word)))", "(word >> (bits * (per_word - 1 - k % per_word)))"),
    "bits_mask_one_bit_short": ("((1u << bits) - 1u)", "((1u << (bits - 1)) - 1u)"),
    "bits_word_stride_of_4_bits": ("wq[n * (K / per_word) + k / per_word]", "wq[n * (K / 8) + k / per_word]"),
    "bits_eight_per_word": ("const int64_t per_word = 32 / bits;", "const int64_t per_word = 8;"),
    "bits_ignored": ("(float)unpack_code_bits(wq, K, n, k, bits)", "(float)unpack_code_bits(wq, K, n, k, 4)"),
}

# Mistakes planted only in the b-bit dot product (its text repeats the 4-bit one's): the
# first occurrence after the anchor is replaced.
BITS_ANCHOR = "static float dot_fp32_bits("
BITS_MUTANTS = {
    "bits_bias_dropped": ("const float w = sq + bi;", "const float w = sq;"),
    "bits_scale_dropped": ("const float sq = sc * q;", "const float sq = q;"),
    "bits_scale_group_index": ("bf16_to_f32(s[n * G + k / 128])", "bf16_to_f32(s[n * G + (k / 128) % 1])"),
    "bits_x_index": ("x[m * K + k]", "x[m * K + (k ^ 1)]"),
    "bits_fp64_accumulator": ("float acc = 0.0f;", "double acc = 0.0;"),
    "bits_k_descending": ("for (int64_t k = 0; k < K; ++k) {", "for (int64_t k = K - 1; k >= 0; --k) {"),
}


def _build(tmp_path, name, src_text, extra_flags=()):
    src = tmp_path / f"{name}.c"
    src.write_text(src_text)
    out = tmp_path / f"lib{name}.so"
    flags = [f for f in oracle.CFLAGS if f != "-Werror"]   # a mutant may leave a variable unused
    subprocess.run(["gcc", *flags, *extra_flags, str(src), "-o", str(out), *oracle.LIBS], check=True)
    return str(out)


def _run_pins(lib):
    env = dict(os.environ)
    env["PYTHONPATH"] = os.pathsep.join([os.path.dirname(HERE), HERE, env.get("PYTHONPATH", "")])
    env["OMP_NUM_THREADS"] = "1"
    r = subprocess.run([sys.executable, os.path.join(HERE, "oracle_pins.py"), lib],
                       capture_output=True, text=True, timeout=600, env=env)
    return r.returncode, r.stdout + r.stderr


def test_real_source_passes(tmp_path):
    lib = _build(tmp_path, "real", open(oracle.SOURCE).read())
    rc, out = _run_pins(lib)
    assert rc == 0, out


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, name):
    old, new = MUTANTS[name]
    text = open(oracle.SOURCE).read()
    assert old in text, f"mutation site for {name} not found"
    lib = _build(tmp_path, name, text.replace(old, new))
    rc, out = _run_pins(lib)
    assert rc != 0, f"{name} survived every pin: {out}"


@pytest.mark.parametrize("name", sorted(BITS_MUTANTS))
def test_bits_mutant_is_caught(tmp_path, name):
    old, new = BITS_MUTANTS[name]
    text = open(oracle.SOURCE).read()
    a = text.index(BITS_ANCHOR)
    i = text.index(old, a)
    lib = _build(tmp_path, name, text[:i] + new + text[i + len(old):])
    rc, out = _run_pins(lib)
    assert rc != 0 and "pin_bits" in out, f"{name} survived the b-bit pins: {out}"


def test_fused_multiply_add_is_caught(tmp_path):
    """Building with contraction into FMAs must trip the unfused-product pin."""
    try:
        lib = _build(tmp_path, "fused", open(oracle.SOURCE).read(),
                     extra_flags=("-ffp-contract=fast", "-mfma"))
    except subprocess.CalledProcessError:
        pytest.skip("compiler cannot target FMA here")
    rc, out = _run_pins(lib)
    assert rc != 0 and "pin_matmul_golden_cases" in out, out
