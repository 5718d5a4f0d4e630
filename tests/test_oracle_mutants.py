"""Planted mistakes: every plausible slip in the oracle must fail a pin.

Each case below copies ``oracle/far_oracle.c``, applies one textual change
that models a plausible mistake (a dropped term, a wrong divisor, a wrong
index, a wrong rounding rule, ...), compiles the copy into a temporary
directory, points the oracle wrapper at it and runs a quick subset of the
pins in ``test_oracle_pins.py``.  At least one pin must fail for every
mutant; the real oracle must pass the same subset.  Only the CPU and the
oracle are involved.
"""
from __future__ import annotations

import subprocess

import pytest

import oracle
import oracle.build as obuild
import test_oracle_pins as pins

SRC = open(obuild.SRC).read()

MUTANTS = {
    "residual dropped": ("s += far_oracle_decode16(residual[base + h], dtype);", "s += 0.0;"),
    "last partial dropped": ("for (int r = 0; r < W; ++r)", "for (int r = 0; r < W - 1; ++r)"),
    "partial column shifted": ("partials[r][base + h]", "partials[r][base + (h + r) % H]"),
    "mean over H-1": ("ss / (double)H", "ss / (double)(H - 1)"),
    "eps outside the root": ("1.0 / sqrt(ms + (double)eps)", "1.0 / (sqrt(ms) + (double)eps)"),
    "eps dropped": ("1.0 / sqrt(ms + (double)eps)", "1.0 / sqrt(ms)"),
    "rms instead of 1/rms": ("1.0 / sqrt(ms + (double)eps)", "sqrt(ms + (double)eps)"),
    "eps in double, not its fp32 value": ("1.0 / sqrt(ms + (double)eps)", "1.0 / sqrt(ms + (eps == 1e-6f ? 1e-6 : (double)eps))"),
    "weight_bias ignored": ("far_oracle_decode16(gamma[h], dtype) + (double)weight_bias", "far_oracle_decode16(gamma[h], dtype) + 0.0"),
    "weight_bias subtracted": ("far_oracle_decode16(gamma[h], dtype) + (double)weight_bias", "far_oracle_decode16(gamma[h], dtype) - (double)weight_bias"),
    "gamma reversed": ("gamma[h]", "gamma[H - 1 - h]"),
    "row offset relative to the slice": ("        const int64_t base = t * H;\n        const double rinv = row_y_o(",
                                         "        const int64_t base = (t - row_begin) * H;\n        const double rinv = row_y_o("),
    "16-bit rounding truncates": ("double v = nearbyint(a / quantum) * quantum; /* a/quantum is exact */",
                                  "double v = floor(a / quantum) * quantum;"),
    "16-bit subnormals flushed": ("    if (be < f.emin)\n        be = f.emin;       /* below the normal range the spacing is fixed */\n",
                                  "    if (be < f.emin)\n        return sign;\n"),
    "fp16 bias off by one": ("f.mbits = 10; f.ebits = 5; f.bias = 15;", "f.mbits = 10; f.ebits = 5; f.bias = 16;"),
    "e4m3 ties away from zero": ("    double v = nearbyint(a / quantum) * quantum;\n    if (v > 448.0)",
                                 "    double v = round(a / quantum) * quantum;\n    if (v > 448.0)"),
    "e4m3 overflow to NaN": ("return (uint8_t)(sign | 0x7E);        /* S.1111.110 = 448 */", "return 0x7F;"),
    "e4m3 subnormal step": ("    if (be < -6)\n        be = -6;                               /* subnormal spacing 2^-9 */",
                            "    if (be < -7)\n        be = -7;"),
    "static scale multiplied": ("to_f32(to_f32(o[h]) / s32)", "to_f32(to_f32(o[h]) * s32)"),
    "e4m3fnuz maximum 240": ("double scale = to_f32(amax / 448.0);", "double scale = to_f32(amax / 240.0);"),
    "amax without abs": ("double a = fabs(to_f32(o[h]));", "double a = to_f32(o[h]);"),
    "static code decided in fp64": ("far_oracle_e4m3_encode(to_f32(to_f32(o[h]) / s32))", "far_oracle_e4m3_encode(o[h] / s32)"),
    "dynamic code decided in fp64": ("far_oracle_e4m3_encode(to_f32(to_f32(o[h]) / scale))", "far_oracle_e4m3_encode(o[h] / scale)"),
    "per-tensor code decided in fp64": ("far_oracle_e4m3_encode(to_f32(to_f32(o[h]) / tensor_scale))", "far_oracle_e4m3_encode(o[h] / tensor_scale)"),
    "per-tensor amax of the first row only": ("            row_y_o(partials, W, residual, gamma, t, H, dtype, eps, weight_bias, acc32, y, o);\n            for (int64_t h = 0; h < H; ++h) {",
                                              "            row_y_o(partials, W, residual, gamma, t, H, dtype, eps, weight_bias, acc32, y, o);\n            if (t > row_begin) break;\n            for (int64_t h = 0; h < H; ++h) {"),
    "fp32 accumulation kept in fp64": ("            float s = 0.0f; /* 2-byte values convert to float exactly */",
                                       "            double s = 0.0f; /* 2-byte values convert to float exactly */"),
    "fp32 accumulation drops the residual": ("                s = s + (float)far_oracle_decode16(residual[base + h], dtype);",
                                             "                s = s + 0.0f;"),
    "per-tensor scale over 240": ("tensor_scale = to_f32(amax / 448.0);", "tensor_scale = to_f32(amax / 240.0);"),
    "per-group amax over the first group only": ("for (int64_t h = q * group; h < (q + 1) * group; ++h) {\n                    double a", "for (int64_t h = 0; h < group; ++h) {\n                    double a"),
    "per-group scales indexed by group only": ("scale_out[t * ngroups + q] = (float)scale;", "scale_out[q] = (float)scale;"),
    "y squared without the residual": ("ss += y[h] * y[h];", "ss += (y[h] - (residual ? far_oracle_decode16(residual[base + h], dtype) : 0.0)) * (y[h] - (residual ? far_oracle_decode16(residual[base + h], dtype) : 0.0));"),
}


def quick_pins():
    """A subset of the pins that runs in a second or two."""
    for dt in ("bf16", "fp16"):
        for pattern in (0, 1, 2, 3):
            for shape in ((2, 8, 4), (3, 5, 4), (1, 4, 32)):
                yield "brute force %s %s %s" % (shape, pattern, dt), lambda s=shape, p=pattern, d=dt: pins.test_brute_force_exact_tiny(s, p, d)
    for pattern in (0, 1, 2, 3):
        yield "brute force gemma / no residual %d" % pattern, lambda p=pattern: pins.test_brute_force_exact_gemma_and_no_residual(p)
    yield "worked standard + static", pins.test_worked_example_standard_and_static_fp8
    yield "worked gemma + dynamic", pins.test_worked_example_gemma_and_dynamic_fp8
    yield "worked tie to even", pins.test_worked_example_fp8_tie_to_even
    yield "worked fp32 decision", pins.test_worked_example_fp8_code_decided_in_fp32
    yield "worked fp32 decision dynamic", pins.test_worked_example_dynamic_fp8_code_decided_in_fp32
    yield "worked per-tensor", pins.test_worked_example_per_tensor_fp8
    yield "worked per-group", pins.test_worked_example_per_group_fp8
    for dt in ("bf16", "fp16"):
        yield "per-group invariants %s" % dt, lambda d=dt: pins.test_per_group_invariants(d)
    yield "brute force per-group", lambda: pins.test_brute_force_exact_per_group((2, 8, 64), 16, "bf16")
    for dt in ("bf16", "fp16"):
        yield "per-tensor vs per-token %s" % dt, lambda d=dt: pins.test_per_tensor_scale_is_the_largest_per_token_scale(d)
    yield "worked zeros", pins.test_worked_example_zero_input_scale_one
    yield "worked saturation", pins.test_worked_example_saturation_and_zero_row_dynamic
    for dt in ("bf16", "fp16"):
        yield "round16 specials %s" % dt, lambda d=dt: pins.test_round16_overflow_and_specials(d)
    yield "e4m3 codes", pins.test_e4m3_all_codes_decode_and_roundtrip
    yield "e4m3 midpoints", pins.test_e4m3_midpoints_ties_to_even_and_saturation
    yield "one rank", pins.test_one_rank_is_plain_add_rmsnorm
    yield "rms one", pins.test_rms_of_output_is_one_within_eps
    yield "gemma", pins.test_gemma_weight_bias_equals_gamma_plus_one
    yield "first pattern", pins.test_first_pattern_without_residual
    yield "gamma column", pins.test_gamma_is_indexed_by_column
    yield "order", pins.test_partial_order_does_not_matter
    yield "fp32 accumulation worked example", pins.test_worked_example_fp32_accumulation
    for pattern in (0, 2):
        yield "fp32 accumulation exact when the sum is %d" % pattern, lambda p=pattern: pins.test_fp32_accumulation_equals_exact_without_cancellation(p)


def run_quick_pins():
    """Names of the quick pins that fail."""
    failed = []
    for name, fn in quick_pins():
        try:
            fn()
        except (AssertionError, ValueError):
            failed.append(name)
    return failed


def test_real_oracle_passes_quick_pins():
    assert run_quick_pins() == []


def test_row_slice_pin_catches_relative_offset(tmp_path, monkeypatch):
    # the row-offset mutant only shows on a slice that does not start at 0,
    # which the row-slice pin covers; run it alone since it is larger
    _with_mutant(tmp_path, monkeypatch, "row offset relative to the slice")
    with pytest.raises(AssertionError):
        pins.test_row_slices_equal_full_rows()


def _with_mutant(tmp_path, monkeypatch, name):
    old, new = MUTANTS[name]
    assert SRC.count(old) >= 1, "mutation target vanished from the oracle: %r" % old
    src = tmp_path / "mutant.c"
    src.write_text(SRC.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", *obuild.CFLAGS, "-o", str(lib), str(src), "-lm"],
                   check=True, capture_output=True)
    monkeypatch.setattr(oracle, "_lib", oracle.load(str(lib)))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_fails_a_pin(name, tmp_path, monkeypatch):
    _with_mutant(tmp_path, monkeypatch, name)
    if name == "row offset relative to the slice":
        with pytest.raises(AssertionError):
            pins.test_row_slices_equal_full_rows()
        return
    failed = run_quick_pins()
    assert failed, "planted mistake %r passed every quick pin" % name
