"""Pins for the fp64 CPU oracle, against things other than itself.

The pages print no numeric worked example, so the oracle is pinned by:
exact-rational brute force on tiny shapes (Fraction arithmetic, one square
root bracketed with 60-digit decimal), hand-derived closed-form cases, the
format definitions (checked exhaustively and against torch's CPU casts, a
library routine used only as a check), and the invariants the pages state:

* the result is norm(all_reduce(h), residual) and the new residual is
  all_reduce(h) + residual [vllm.models.common.ops.fused_allreduce_rms_norm,
  docstring of fused_allreduce_rms_norm];
* one rank is the plain fused add + RMSNorm [same page, tp_size == 1 branch];
* weight_bias 0.0 is standard RMSNorm, 1.0 is Gemma-style gamma + 1 [same
  page, the weight_bias argument];
* ReduceScatter -> local RMSNorm -> AllGather equals the full-row result
  [vllm.compilation.sequence_parallelism, SequenceParallelismPass docstring];
* a 3-D [batch, tokens, hidden] input equals its 2-D view [PR #45307 report,
  call_trtllm_fused_allreduce_norm];
* dynamic per-token FP8 returns one scale per token, scale = amax / 448 for
  e4m3 [vllm.compilation.fusion, FusedAddRMSNormDynamicQuantPattern].
"""
from __future__ import annotations

import math
import struct
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from exact_ref import (INF, decode, e4m3_sat, encode, f32, inv_sqrt_bracket,
                       rne, rne_bracket)
from reduce_residual_add_b200.inputs import WORKLOADS, as_u16, make_inputs, random_inputs


def zero_sign_free(a: np.ndarray) -> np.ndarray:
    """Map the negative-zero pattern onto +0 (the sign of a zero is not compared)."""
    a = a.copy()
    if a.dtype == np.uint16:
        a[a == 0x8000] = 0
    elif a.dtype == np.uint8:
        a[a == 0x80] = 0
    return a


# ---------------------------------------------------------------------------
# number formats
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("dt", ["bf16", "fp16"])
def test_decode16_all_patterns_match_definition_and_torch(dt):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    tdt = torch.bfloat16 if dt == "bf16" else torch.float16
    via_torch = torch.from_numpy(bits.view(np.int16)).view(tdt).to(torch.float64).numpy()
    L = oracle.lib()
    code = oracle.dtype_code(dt)
    for b in range(0, 65536, 1):
        v = L.far_oracle_decode16(b, code)
        ex = decode(b, dt)
        if ex is None:
            assert math.isnan(v) and math.isnan(via_torch[b])
        else:
            assert v == float(ex) == via_torch[b], hex(b)


@pytest.mark.parametrize("dt", ["bf16", "fp16"])
def test_round16_exhaustive_midpoints_ties_to_even(dt):
    """Every midpoint between adjacent finite values rounds to the even pattern,
    and the doubles just either side of it round down / up."""
    L = oracle.lib()
    code = oracle.dtype_code(dt)
    maxbits = 0x7F7F if dt == "bf16" else 0x7BFF
    for b in range(0, maxbits):
        lo, hi = decode(b, dt), decode(b + 1, dt)
        mid = (lo + hi) / 2
        m = float(mid)
        assert Fraction(m) == mid          # representable in a double
        want = b if b % 2 == 0 else b + 1
        assert L.far_oracle_round16(m, code) == want, hex(b)
        assert L.far_oracle_round16(-m, code) == want | 0x8000
        assert L.far_oracle_round16(math.nextafter(m, -INF), code) == b
        assert L.far_oracle_round16(math.nextafter(m, INF), code) == b + 1
        assert L.far_oracle_round16(float(lo), code) == b


@pytest.mark.parametrize("dt", ["bf16", "fp16"])
def test_round16_overflow_and_specials(dt):
    L = oracle.lib()
    code = oracle.dtype_code(dt)
    maxbits = 0x7F7F if dt == "bf16" else 0x7BFF
    inf_bits = 0x7F80 if dt == "bf16" else 0x7C00
    top = decode(maxbits, dt)
    ulp = top - decode(maxbits - 1, dt)
    # the midpoint above the largest finite value ties to the even "next"
    # binade, i.e. overflows to infinity; just below it stays finite
    m = float(top + ulp / 2)
    assert L.far_oracle_round16(m, code) == inf_bits
    assert L.far_oracle_round16(math.nextafter(m, 0), code) == maxbits
    assert L.far_oracle_round16(-m, code) == inf_bits | 0x8000
    assert L.far_oracle_round16(INF, code) == inf_bits
    assert L.far_oracle_round16(0.0, code) == 0
    assert L.far_oracle_round16(-0.0, code) == 0x8000
    nan = L.far_oracle_round16(float("nan"), code)
    assert decode(nan, dt) is None
    # below half the smallest subnormal: zero; at half: tie to even zero
    tiny = decode(1, dt)
    assert L.far_oracle_round16(float(tiny / 2), code) == 0
    assert L.far_oracle_round16(float(tiny * 3 / 4), code) == 1
    assert L.far_oracle_round16(float(tiny * 3 / 2), code) == 2


@pytest.mark.parametrize("dt", ["bf16", "fp16"])
def test_round16_matches_torch_cast_from_fp32(dt):
    """Single rounding fp32 -> 16-bit: the oracle agrees with torch's cast."""
    g = torch.Generator().manual_seed(11)
    x = torch.randn(200000, generator=g, dtype=torch.float32)
    e = torch.randint(-30, 20, (200000,), generator=g).to(torch.float32)
    x = x * torch.exp2(e)
    if dt == "fp16":
        x = x.clamp(-60000, 60000)
    tdt = torch.bfloat16 if dt == "bf16" else torch.float16
    want = as_u16(x.to(tdt))
    L = oracle.lib()
    code = oracle.dtype_code(dt)
    xs = x.numpy().astype(np.float64)
    got = np.array([L.far_oracle_round16(float(v), code) for v in xs], dtype=np.uint16)
    np.testing.assert_array_equal(got, want)


def test_e4m3_all_codes_decode_and_roundtrip():
    L = oracle.lib()
    for c in range(256):
        ex = decode(c, "e4m3")
        v = L.far_oracle_e4m3_decode(c)
        if ex is None:
            assert math.isnan(v)
            assert c in (0x7F, 0xFF)
            continue
        assert v == float(ex)
        back = L.far_oracle_e4m3_encode(v)
        if c == 0x80:
            assert back == 0x80            # -0 keeps its sign
        else:
            assert back == c, (hex(c), hex(back))
    assert float(decode(0x7E, "e4m3")) == 448.0
    assert float(decode(0x01, "e4m3")) == 2.0 ** -9
    assert float(decode(0x08, "e4m3")) == 2.0 ** -6


def test_e4m3_midpoints_ties_to_even_and_saturation():
    L = oracle.lib()
    for c in range(0, 0x7E):
        lo, hi = decode(c, "e4m3"), decode(c + 1, "e4m3")
        mid = float((lo + hi) / 2)
        want = c if c % 2 == 0 else c + 1
        assert L.far_oracle_e4m3_encode(mid) == want, hex(c)
        assert L.far_oracle_e4m3_encode(-mid) == want | 0x80
        assert L.far_oracle_e4m3_encode(math.nextafter(mid, -INF)) == c
        assert L.far_oracle_e4m3_encode(math.nextafter(mid, INF)) == c + 1
    # satfinite: everything at or beyond 448 in magnitude maps to +-448
    for v in (448.0, 448.0001, 464.0, 479.9, 480.0, 1e6, 1e300, INF):
        assert L.far_oracle_e4m3_encode(v) == 0x7E
        assert L.far_oracle_e4m3_encode(-v) == 0xFE
    assert L.far_oracle_e4m3_encode(float("nan")) == 0x7F
    # below half the smallest subnormal rounds to zero; exactly half ties to 0
    assert L.far_oracle_e4m3_encode(2.0 ** -10) == 0x00
    assert L.far_oracle_e4m3_encode(math.nextafter(2.0 ** -10, 1)) == 0x01


def test_e4m3_matches_torch_cast_in_range():
    """torch's float8_e4m3fn cast (round to nearest even, no saturation) agrees
    with the oracle for every fp32 input of magnitude below 448."""
    g = torch.Generator().manual_seed(5)
    x = torch.randn(300000, generator=g) * torch.exp2(torch.randint(-12, 9, (300000,), generator=g).float())
    x = x.clamp(-447.99, 447.99)
    want = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    L = oracle.lib()
    got = np.array([L.far_oracle_e4m3_encode(float(v)) for v in x.numpy()], dtype=np.uint8)
    np.testing.assert_array_equal(got, want)


# ---------------------------------------------------------------------------
# exact-rational brute force of the whole epilogue
# ---------------------------------------------------------------------------

def exact_fused(ps, res, gam, dt, eps, wb, pattern, scale_in=None, group=0):
    """Fraction-exact epilogue on bit patterns (lists of rows of ints)."""
    T, H = len(ps[0]), len(gam)
    epsq, wbq = f32(eps), f32(wb)
    g = [decode(int(b), dt) + wbq for b in gam]
    out = {"residual_out": [], "norm_out": [], "quant_out": [], "scale_out": []}
    rows = []
    for t in range(T):
        y = []
        for h in range(H):
            s = sum(decode(int(p[t][h]), dt) for p in ps)
            if res is not None:
                s += decode(int(res[t][h]), dt)
            y.append(s)
        ms = sum(v * v for v in y) / H
        rlo, rhi = inv_sqrt_bracket(ms + epsq)
        o_lo, o_hi = [], []
        for h in range(H):
            a, b = y[h] * g[h] * rlo, y[h] * g[h] * rhi
            o_lo.append(min(a, b))
            o_hi.append(max(a, b))
        out["residual_out"].append([encode(rne(v, dt), dt) for v in y])
        row_norm = []
        for lo, hi in zip(o_lo, o_hi):
            r = rne_bracket(lo, hi, dt)
            row_norm.append(None if r is None else encode(r, dt))
        out["norm_out"].append(row_norm)
        o32 = [rne_bracket(lo, hi, "fp32") for lo, hi in zip(o_lo, o_hi)]
        if pattern == oracle.FP8_STATIC:
            s32 = f32(scale_in)
            out["quant_out"].append([None if v is None else encode(e4m3_sat(rne(v / s32, "fp32")), "e4m3")
                                     for v in o32])
        elif pattern == oracle.FP8_TOKEN:
            assert all(v is not None for v in o32)
            amax = max(abs(v) for v in o32)
            sc = rne(amax / 448, "fp32")
            out["scale_out"].append(sc)
            if sc == 0:
                out["quant_out"].append([0] * H)
            else:
                out["quant_out"].append([encode(e4m3_sat(rne(v / sc, "fp32")), "e4m3") for v in o32])
        elif pattern == oracle.FP8_GROUP:
            assert all(v is not None for v in o32)
            codes = []
            for q in range(H // group):
                chunk = o32[q * group:(q + 1) * group]
                sc = rne(max(abs(v) for v in chunk) / 448, "fp32")
                out["scale_out"].append(sc)
                codes += [0] * group if sc == 0 else [encode(e4m3_sat(rne(v / sc, "fp32")), "e4m3") for v in chunk]
            out["quant_out"].append(codes)
        rows.append(o32)
    if pattern == oracle.FP8_TENSOR:
        # one scale: amax over every row of the call
        assert all(v is not None for r in rows for v in r)
        amax = max(abs(v) for r in rows for v in r)
        sc = rne(amax / 448, "fp32")
        out["scale_out"] = [sc]
        for r in rows:
            out["quant_out"].append([0] * H if sc == 0 else
                                    [encode(e4m3_sat(rne(v / sc, "fp32")), "e4m3") for v in r])
    return out


def _compare_exact(inp, dt, eps, wb, pattern, scale_in=None, group=0):
    ps = [as_u16(p) for p in inp["partials"]]
    res = None if inp["residual"] is None else as_u16(inp["residual"])
    gam = as_u16(inp["gamma"])
    got = oracle.fused(ps, res, gam, dt, eps, wb, pattern, scale_in=scale_in, group=group)
    ex = exact_fused([p.tolist() for p in ps], None if res is None else res.tolist(),
                     gam.tolist(), dt, eps, wb, pattern, scale_in, group)
    np.testing.assert_array_equal(zero_sign_free(got["residual_out"]),
                                  zero_sign_free(np.array(ex["residual_out"], np.uint16)))
    n_amb = 0
    for t, row in enumerate(ex["norm_out"]):
        for h, v in enumerate(row):
            if v is None:
                n_amb += 1
                continue
            a = int(got["norm_out"][t, h])
            assert (a if a & 0x7FFF else 0) == (v if v & 0x7FFF else 0), (t, h, hex(a), hex(v))
    if pattern != oracle.AR_RESIDUAL_RMSNORM:
        for t, row in enumerate(ex["quant_out"]):
            for h, v in enumerate(row):
                if v is None:
                    n_amb += 1
                    continue
                a = int(got["quant_out"][t, h])
                assert (a if a & 0x7F else 0) == (v if v & 0x7F else 0), (t, h, hex(a), hex(v))
    if pattern in (oracle.FP8_TOKEN, oracle.FP8_TENSOR, oracle.FP8_GROUP):
        flat = got["scale_out"].reshape(-1)
        for t, sc in enumerate(ex["scale_out"]):
            assert Fraction(float(flat[t])) == sc
    assert n_amb == 0


@pytest.mark.parametrize("dt", ["bf16", "fp16"])
@pytest.mark.parametrize("pattern", [0, 1, 2, 3])
@pytest.mark.parametrize("shape", [(2, 8, 4), (1, 5, 4), (3, 5, 4), (2, 8, 64)])
def test_brute_force_exact_tiny(shape, pattern, dt):
    """Tracing shapes [1, 8, 4] (sequence_parallelism patterns), (5, 4)
    (fusion patterns) and the W=2, T=8, H=64 small workload."""
    W, T, H = shape
    inp = random_inputs(W, T, H, dtype=dt, seed=100 + W * 7 + T + H + pattern)
    _compare_exact(inp, dt, eps=1e-6, wb=0.0, pattern=pattern, scale_in=0.05)


@pytest.mark.parametrize("dt", ["bf16", "fp16"])
@pytest.mark.parametrize("shape,group", [((2, 8, 4), 2), ((3, 5, 16), 8), ((2, 8, 64), 16), ((1, 4, 32), 32)])
def test_brute_force_exact_per_group(shape, group, dt):
    W, T, H = shape
    inp = random_inputs(W, T, H, dtype=dt, seed=300 + W + T + H + group)
    _compare_exact(inp, dt, eps=1e-6, wb=0.0, pattern=oracle.FP8_GROUP, group=group)


@pytest.mark.parametrize("pattern", [0, 1, 2, 3])
def test_brute_force_exact_gemma_and_no_residual(pattern):
    inp = random_inputs(2, 6, 16, dtype="bf16", seed=77)
    _compare_exact(inp, "bf16", eps=1e-5, wb=1.0, pattern=pattern, scale_in=0.02)
    inp = random_inputs(3, 6, 16, dtype="bf16", seed=78, has_residual=False)
    _compare_exact(inp, "bf16", eps=1e-6, wb=0.0, pattern=pattern, scale_in=0.02)


def test_brute_force_exact_small_workload():
    wl = WORKLOADS["c1_small"]
    inp = make_inputs(wl)
    _compare_exact(inp, wl.dtype, wl.eps, wl.weight_bias, wl.pattern)


# ---------------------------------------------------------------------------
# hand-derived closed-form cases (every step exact on paper)
# ---------------------------------------------------------------------------

def _bits(vals, dt="bf16"):
    return np.array([encode(Fraction(v), dt) for v in vals], dtype=np.uint16).reshape(1, -1)


def test_worked_example_standard_and_static_fp8():
    # p0 + p1 + residual = y = [3, 2, 1, 1]; sum y^2 = 15, mean 3.75;
    # eps = 0.25 so mean + eps = 4 and rinv = 1/2 exactly;
    # gamma = [1, 0.5, 2, -1], weight_bias 0: o = y/2 * gamma = [1.5, 0.5, 1, -0.5]
    p0, p1, res = [1, 1, 0.5, 2], [1, 0.5, 0.25, -0.5], [1, 0.5, 0.25, -0.5]
    gam = [1, 0.5, 2, -1]
    r = oracle.fused([_bits(p0), _bits(p1)], _bits(res), _bits(gam)[0], "bf16",
                     eps=0.25, weight_bias=0.0, pattern=oracle.FP8_STATIC,
                     scale_in=0.25, debug=True)
    assert r["rinv"][0] == 0.5
    np.testing.assert_array_equal(r["residual_out"], _bits([3, 2, 1, 1]))
    np.testing.assert_array_equal(r["norm_out"], _bits([1.5, 0.5, 1, -0.5]))
    # o / 0.25 = [6, 2, 4, -2]: 6 = 1.5*2^2 -> E=9, M=4 -> 0x4C; 2 -> 0x40;
    # 4 -> 0x48; -2 -> 0xC0
    assert r["quant_out"][0].tolist() == [0x4C, 0x40, 0x48, 0xC0]


def test_worked_example_gemma_and_dynamic_fp8():
    # same y and rinv; gamma = [0, -0.5, 1, 0.5] with weight_bias 1.0 gives
    # multipliers [1, 0.5, 2, 1.5]: o = [1.5, 0.5, 1, 0.75]
    p0, p1, res = [1, 1, 0.5, 2], [1, 0.5, 0.25, -0.5], [1, 0.5, 0.25, -0.5]
    gam = [0, -0.5, 1, 0.5]
    r = oracle.fused([_bits(p0), _bits(p1)], _bits(res), _bits(gam)[0], "bf16",
                     eps=0.25, weight_bias=1.0, pattern=oracle.FP8_TOKEN)
    np.testing.assert_array_equal(r["norm_out"], _bits([1.5, 0.5, 1, 0.75]))
    # amax = 1.5, scale = fp32(1.5 / 448)
    sc = struct.unpack("<f", struct.pack("<f", 1.5 / 448))[0]
    assert r["scale_out"][0] == np.float32(sc)
    # o / scale ~ [448, 149.3, 298.7, 224]: 448 -> 0x7E; 149.3 -> 144
    # (binade [128,256), step 16; 144 = 1.125*2^7 -> 0x71); 298.7 -> 288
    # (step 32; 1.125*2^8 -> 0x79); 224 = 1.75*2^7 -> 0x76
    assert r["quant_out"][0].tolist() == [0x7E, 0x71, 0x79, 0x76]


def test_worked_example_fp8_tie_to_even():
    # y = [2.125, 3, 1.5, 0.25]: sum y^2 = 15.828125, mean 3.95703125;
    # eps = 11/256 = 0.04296875 makes mean + eps = 4, rinv = 1/2;
    # gamma = 1: o = [1.0625, 1.5, 0.75, 0.125]; static scale 1/16:
    # o / s = [17, 24, 12, 2].  17 lies halfway between 16 (M=0) and 18 (M=1)
    # and goes to the even 16 -> 0x58; 24 -> 0x5C; 12 -> 0x54; 2 -> 0x40
    y = [2.125, 3, 1.5, 0.25]
    r = oracle.fused([_bits(y)], None, _bits([1, 1, 1, 1])[0], "bf16",
                     eps=11 / 256, weight_bias=0.0, pattern=oracle.FP8_STATIC,
                     scale_in=1 / 16, debug=True)
    assert r["rinv"][0] == 0.5
    np.testing.assert_array_equal(r["norm_out"], _bits([1.0625, 1.5, 0.75, 0.125]))
    assert r["quant_out"][0].tolist() == [0x58, 0x5C, 0x54, 0x40]


def test_worked_example_fp8_code_decided_in_fp32():
    # as in the tie case, but eps = 11/256 - 2^-28 (the fp32 just below), so
    # mean + eps = 4 - 2^-28 and rinv = 1/2 * (1 + 2^-31 + ...).  In fp64,
    # o0 = 1.0625 * (1 + 2^-31) lies just above the tie 17/16 and would round
    # to 18 (0x59); rounded to fp32 it is exactly 1.0625, the tie, which goes
    # to the even 16 (0x58).  The code is decided in fp32.
    eps = 11 / 256 - 2.0 ** -28
    assert float(np.float32(eps)) == eps
    y = [2.125, 3, 1.5, 0.25]
    r = oracle.fused([_bits(y)], None, _bits([1, 1, 1, 1])[0], "bf16",
                     eps=eps, weight_bias=0.0, pattern=oracle.FP8_STATIC,
                     scale_in=1 / 16, debug=True)
    assert r["o"][0, 0] > 1.0625 and np.float32(r["o"][0, 0]) == np.float32(1.0625)
    assert r["quant_out"][0, 0] == 0x58
    np.testing.assert_array_equal(r["norm_out"], _bits([1.0625, 1.5, 0.75, 0.125]))


def test_worked_example_dynamic_fp8_code_decided_in_fp32():
    # y = [3.5, 17/128, 1.5, 1]: sum y^2 = 254241/16384; eps = 7903/65536 -
    # 2^-27 (an fp32) gives mean + eps = 4 - 2^-27, rinv = 1/2 (1 + 2^-30 + ...).
    # fp32(o) = [1.75, 17/256, 0.75, 0.5]; amax = 1.75, scale = 1.75/448 =
    # 2^-8 exactly; o/scale = [448, 17, 192, 128].  fp64 o1 * 256 lies just
    # above the tie 17 (would give 18, 0x59); in fp32 it is the tie and goes to
    # the even 16 (0x58).  448 -> 0x7E; 192 = 1.5*2^7 -> 0x74; 128 -> 0x70.
    eps = 7903 / 65536 - 2.0 ** -27
    assert float(np.float32(eps)) == eps
    y = [3.5, 17 / 128, 1.5, 1.0]
    r = oracle.fused([_bits(y)], None, _bits([1, 1, 1, 1])[0], "bf16",
                     eps=eps, weight_bias=0.0, pattern=oracle.FP8_TOKEN, debug=True)
    assert r["scale_out"][0] == np.float32(2.0 ** -8)
    assert r["o"][0, 1] * 256 > 17
    assert r["quant_out"][0].tolist() == [0x7E, 0x58, 0x74, 0x70]


def test_worked_example_per_tensor_fp8():
    # two rows with the eps of the dynamic example (mean + eps = 4 - 2^-27,
    # rinv = 1/2 (1 + 2^-30 + ...)): row 0 = [3.5, 17/128, 1.5, 1], row 1 =
    # [-1, 1.5, 3.5, -17/128].  fp32(o): [1.75, 17/256, 0.75, 0.5] and
    # [-0.5, 0.75, 1.75, -17/256]; the tensor amax is 1.75 and the one scale
    # 1.75/448 = 2^-8.  o/scale: [448, 17, 192, 128] -> 0x7E, 0x58 (the tie
    # 17 goes to the even 16 in fp32; fp64 would give 18), 0x74, 0x70; and
    # [-128, 192, 448, -17] -> 0xF0, 0x74, 0x7E, 0xD8.
    eps = 7903 / 65536 - 2.0 ** -27
    rows = np.concatenate([_bits([3.5, 17 / 128, 1.5, 1.0]), _bits([-1.0, 1.5, 3.5, -17 / 128])])
    r = oracle.fused([rows], None, _bits([1, 1, 1, 1])[0], "bf16", eps=eps,
                     pattern=oracle.FP8_TENSOR)
    assert r["scale_out"].tolist() == [2.0 ** -8]
    assert r["quant_out"][0].tolist() == [0x7E, 0x58, 0x74, 0x70]
    assert r["quant_out"][1].tolist() == [0xF0, 0x74, 0x7E, 0xD8]


@pytest.mark.parametrize("dt", ["bf16", "fp16"])
def test_per_tensor_scale_is_the_largest_per_token_scale(dt):
    """max_t fp32(amax_t / 448) = fp32(max_t amax_t / 448) (rounding is
    monotonic): the per-tensor scale equals the largest per-token scale bit
    for bit, the row attaining it gets the same codes under both patterns,
    and the tensor holds a +-448 code."""
    wl = WORKLOADS["c5_gemma_fp8_token_%s" % dt].with_(T=40)   # same distributions, 40 rows
    inp = make_inputs(wl)
    args = ([as_u16(p) for p in inp["partials"]], as_u16(inp["residual"]), as_u16(inp["gamma"]),
            dt, wl.eps, wl.weight_bias)
    tok = oracle.fused(*args, oracle.FP8_TOKEN)
    ten = oracle.fused(*args, oracle.FP8_TENSOR)
    assert ten["scale_out"][0] == tok["scale_out"].max()
    t = int(np.argmax(tok["scale_out"]))
    np.testing.assert_array_equal(ten["quant_out"][t], tok["quant_out"][t])
    assert np.any((ten["quant_out"] & 0x7F) == 0x7E)
    # every other row is quantised more coarsely than alone: |codes| never above its own
    assert np.all((ten["quant_out"] & 0x7F) <= (tok["quant_out"] & 0x7F))
    np.testing.assert_array_equal(ten["residual_out"], tok["residual_out"])
    # the row range sets the tensor: rows [10, 20) only
    part = oracle.fused(*args, oracle.FP8_TENSOR, rows=(10, 20))
    assert part["scale_out"][0] == tok["scale_out"][10:20].max()


def test_worked_example_per_group_fp8():
    # the dynamic example's row, groups of 2: fp32(o) = [1.75, 17/256 | 0.75, 0.5].
    # group 0: amax 1.75, scale 2^-8, o/s = [448, 17] -> 0x7E, 0x58 (tie to even
    # in fp32); group 1: amax 0.75, scale fp32(0.75/448), o/s ~ [448, 298.7]
    # -> 0x7E, 0x79 (288 = 1.125*2^8)
    eps = 7903 / 65536 - 2.0 ** -27
    r = oracle.fused([_bits([3.5, 17 / 128, 1.5, 1.0])], None, _bits([1, 1, 1, 1])[0], "bf16",
                     eps=eps, pattern=oracle.FP8_GROUP, group=2)
    s1 = struct.unpack("<f", struct.pack("<f", 0.75 / 448))[0]
    assert r["scale_out"].tolist() == [[2.0 ** -8, s1]]
    assert r["quant_out"][0].tolist() == [0x7E, 0x58, 0x7E, 0x79]


@pytest.mark.parametrize("dt", ["bf16", "fp16"])
def test_per_group_invariants(dt):
    """One group spanning the row is per-token FP8, bit for bit; with smaller
    groups each row's largest group scale is its per-token scale, and every
    group holds a +-448 code."""
    wl = WORKLOADS["c5_gemma_fp8_token_%s" % dt].with_(T=24)
    inp = make_inputs(wl)
    args = ([as_u16(p) for p in inp["partials"]], as_u16(inp["residual"]), as_u16(inp["gamma"]),
            dt, wl.eps, wl.weight_bias)
    tok = oracle.fused(*args, oracle.FP8_TOKEN)
    whole = oracle.fused(*args, oracle.FP8_GROUP, group=wl.H)
    np.testing.assert_array_equal(whole["quant_out"], tok["quant_out"])
    np.testing.assert_array_equal(whole["scale_out"][:, 0], tok["scale_out"])
    g128 = oracle.fused(*args, oracle.FP8_GROUP, group=128)
    assert g128["scale_out"].shape == (24, wl.H // 128)
    np.testing.assert_array_equal(g128["scale_out"].max(axis=1), tok["scale_out"])
    q = (g128["quant_out"] & 0x7F).reshape(24, wl.H // 128, 128)
    assert np.all(np.any(q == 0x7E, axis=2))
    np.testing.assert_array_equal(g128["residual_out"], tok["residual_out"])


def test_worked_example_zero_input_scale_one():
    # the tracing inputs of the sequence-parallel static-FP8 "First" pattern:
    # an all-zero [1, 8, 4] input and a scale of 1.0.  y = 0, so o = 0 and
    # every code is 0; rinv = 1/sqrt(eps).
    z = np.zeros((1, 8, 4), np.uint16)
    for eps in (1e-5, 1e-6):
        r = oracle.fused([z, z], None, _bits([1, 1, 1, 1])[0], "bf16", eps=eps,
                         pattern=oracle.FP8_STATIC, scale_in=1.0, debug=True)
        assert not r["norm_out"].any() and not r["quant_out"].any()
        assert not r["residual_out"].any()
        assert r["rinv"][0] == 1 / math.sqrt(float(np.float32(eps)))


def test_worked_example_saturation_and_zero_row_dynamic():
    # static: o = [1.5, 0.5, 1, -0.5] with scale 2^-9: o/s = [768, 256, 512,
    # -256]: 768 and 512 saturate to 448 (0x7E), 256 = 2^8 -> 0x78, -256 -> 0xF8
    p0, p1, res = [1, 1, 0.5, 2], [1, 0.5, 0.25, -0.5], [1, 0.5, 0.25, -0.5]
    gam = [1, 0.5, 2, -1]
    r = oracle.fused([_bits(p0), _bits(p1)], _bits(res), _bits(gam)[0], "bf16",
                     eps=0.25, pattern=oracle.FP8_STATIC, scale_in=2.0 ** -9)
    assert r["quant_out"][0].tolist() == [0x7E, 0x78, 0x7E, 0xF8]
    # dynamic on an all-zero row: scale 0 and codes 0
    z = np.zeros((2, 4), np.uint16)
    r = oracle.fused([z], z, _bits(gam)[0], "bf16", eps=1e-6, pattern=oracle.FP8_TOKEN)
    assert r["scale_out"].tolist() == [0.0, 0.0]
    assert not r["quant_out"].any()


# ---------------------------------------------------------------------------
# invariants stated by the pages
# ---------------------------------------------------------------------------

def np_rne16(x: np.ndarray, dt: str) -> np.ndarray:
    """Round float64 -> 16-bit patterns by integer manipulation of the double's
    bits (a second, independent rounding routine; normal range, plus the fp16
    subnormal range by scaling)."""
    x = np.asarray(x, np.float64)
    drop = 45 if dt == "bf16" else 42
    b = x.view(np.uint64).copy()
    lsb = (b >> np.uint64(drop)) & np.uint64(1)
    b = b + (np.uint64(1) << np.uint64(drop - 1)) - np.uint64(1) + lsb
    b &= ~((np.uint64(1) << np.uint64(drop)) - np.uint64(1))
    r = b.view(np.float64)
    if dt == "fp16":
        small = np.abs(x) < 2.0 ** -14
        r = np.where(small, np.rint(x * 2.0 ** 24) * 2.0 ** -24, r)
        return as_u16(torch.from_numpy(r).to(torch.float32).to(torch.float16))
    return as_u16(torch.from_numpy(r).to(torch.float32).to(torch.bfloat16))


def _dec(a: np.ndarray, dt: str) -> np.ndarray:
    tdt = torch.bfloat16 if dt == "bf16" else torch.float16
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(tdt).to(torch.float64).numpy()


def test_one_rank_is_plain_add_rmsnorm():
    """W=1: the oracle equals an independently written numpy fp64 fused
    add + RMSNorm (tp_size == 1 branch of fused_allreduce_rms_norm)."""
    inp = random_inputs(1, 64, 512, seed=21)
    p, res, gam = as_u16(inp["partials"][0]), as_u16(inp["residual"]), as_u16(inp["gamma"])
    eps = 1e-6
    r = oracle.fused([p], res, gam, "bf16", eps, 0.0, debug=True)
    x = _dec(p, "bf16") + _dec(res, "bf16")
    var = np.mean(x * x, axis=-1, keepdims=True)
    o = x / np.sqrt(var + np.float64(np.float32(eps))) * _dec(gam, "bf16")
    np.testing.assert_allclose(r["o"], o, rtol=1e-14, atol=0)
    np.testing.assert_array_equal(zero_sign_free(r["norm_out"]), zero_sign_free(np_rne16(o, "bf16")))
    np.testing.assert_array_equal(r["residual_out"], np_rne16(x, "bf16"))


@pytest.mark.parametrize("name", ["c3_3d", "c5_gemma_fp8_token_fp16"])
def test_new_residual_contract_bitwise(name):
    """residual_out == RNE(sum_r p_r + residual), bit for bit."""
    wl = WORKLOADS[name]
    inp = make_inputs(wl, rows=64)
    ps = [as_u16(p) for p in inp["partials"]]
    res = as_u16(inp["residual"])
    r = oracle.fused(ps, res, as_u16(inp["gamma"]), wl.dtype, wl.eps,
                     wl.weight_bias, wl.pattern, scale_in=wl.static_scale)
    s = sum(_dec(p, wl.dtype) for p in ps) + _dec(res, wl.dtype)
    np.testing.assert_array_equal(zero_sign_free(r["residual_out"]), zero_sign_free(np_rne16(s, wl.dtype)))


def test_new_residual_contract_outlier_rows():
    wl = WORKLOADS["c4_prefill_fp8_static"].with_(T=512)
    inp = make_inputs(wl)
    assert len(inp["outlier_rows"]) == 6
    ps = [as_u16(p) for p in inp["partials"]]
    res = as_u16(inp["residual"])
    r = oracle.fused(ps, res, as_u16(inp["gamma"]), "bf16", wl.eps, 0.0,
                     wl.pattern, scale_in=wl.static_scale, want_norm=True)
    s = sum(_dec(p, "bf16") for p in ps) + _dec(res, "bf16")
    np.testing.assert_array_equal(zero_sign_free(r["residual_out"]), zero_sign_free(np_rne16(s, "bf16")))


def test_rms_of_output_is_one_within_eps():
    inp = random_inputs(3, 32, 1024, seed=31)
    ones = as_u16(torch.ones(1024, dtype=torch.bfloat16))
    eps = 1e-5
    r = oracle.fused([as_u16(p) for p in inp["partials"]], as_u16(inp["residual"]),
                     ones, "bf16", eps, 0.0, debug=True)
    ms = np.mean(r["y"] ** 2, axis=1)
    e = float(np.float32(eps))
    np.testing.assert_allclose(np.mean(r["o"] ** 2, axis=1), ms / (ms + e), rtol=1e-12)
    assert np.all(np.abs(np.mean(r["o"] ** 2, axis=1) - 1) <= e / ms + 1e-12)


def test_gemma_weight_bias_equals_gamma_plus_one():
    """weight_bias = 1.0 with gamma equals weight_bias = 0 with gamma + 1, for
    gammas whose +1 is exact in bf16 (multiples of 2^-7 in [-1, 1))."""
    g = torch.Generator().manual_seed(41)
    k = torch.randint(-128, 128, (256,), generator=g)
    gam = (k.double() / 128).to(torch.bfloat16)
    gam1 = (k.double() / 128 + 1).to(torch.bfloat16)
    assert torch.equal(gam.double() + 1, gam1.double())
    inp = random_inputs(2, 16, 256, seed=42)
    ps, res = [as_u16(p) for p in inp["partials"]], as_u16(inp["residual"])
    for pattern in (0, 1, 2):
        a = oracle.fused(ps, res, as_u16(gam), "bf16", 1e-6, 1.0, pattern, scale_in=0.03)
        b = oracle.fused(ps, res, as_u16(gam1), "bf16", 1e-6, 0.0, pattern, scale_in=0.03)
        for key in ("residual_out", "norm_out", "quant_out", "scale_out"):
            if a[key] is not None:
                np.testing.assert_array_equal(a[key], b[key])
    # and weight_bias does change the result (it is not ignored)
    c = oracle.fused(ps, res, as_u16(gam), "bf16", 1e-6, 0.0, 0)
    d = oracle.fused(ps, res, as_u16(gam), "bf16", 1e-6, 1.0, 0)
    assert not np.array_equal(c["norm_out"], d["norm_out"])


def test_row_slices_equal_full_rows():
    """ReduceScatter -> local norm -> AllGather: two 512-row slices written
    at their row offsets equal the full 1024-row result."""
    wl = WORKLOADS["c3_3d"]
    inp = make_inputs(wl)
    ps = [as_u16(p) for p in inp["partials"]]
    res, gam = as_u16(inp["residual"]), as_u16(inp["gamma"])
    for pattern in (0, 1, 2):
        full = oracle.fused(ps, res, gam, "bf16", wl.eps, 0.0, pattern, scale_in=0.05)
        parts = oracle.fused(ps, res, gam, "bf16", wl.eps, 0.0, pattern, scale_in=0.05, rows=(0, 512))
        oracle.fused(ps, res, gam, "bf16", wl.eps, 0.0, pattern, scale_in=0.05, rows=(512, 1024), out=parts)
        for key in ("residual_out", "norm_out", "quant_out", "scale_out"):
            if full[key] is not None:
                np.testing.assert_array_equal(full[key], parts[key])


def test_three_d_equals_flat_view():
    wl = WORKLOADS["c3_3d"]
    inp = make_inputs(wl, rows=256)
    ps = [as_u16(p) for p in inp["partials"]]
    res, gam = as_u16(inp["residual"]), as_u16(inp["gamma"])
    flat = oracle.fused(ps, res, gam, "bf16", wl.eps, 0.0, 0)
    three = oracle.fused([p.reshape(4, 64, 2048) for p in ps], res.reshape(4, 64, 2048),
                         gam, "bf16", wl.eps, 0.0, 0)
    np.testing.assert_array_equal(flat["norm_out"], three["norm_out"])
    np.testing.assert_array_equal(flat["residual_out"], three["residual_out"])


@pytest.mark.parametrize("dt", ["bf16", "fp16"])
def test_dynamic_scale_is_amax_over_448(dt):
    wl = WORKLOADS["c5_gemma_fp8_token_%s" % dt]
    inp = make_inputs(wl, rows=48)
    r = oracle.fused([as_u16(p) for p in inp["partials"]], as_u16(inp["residual"]),
                     as_u16(inp["gamma"]), dt, wl.eps, wl.weight_bias, wl.pattern, debug=True)
    amax = np.max(np.abs(r["o"].astype(np.float32)), axis=1)
    want = (amax.astype(np.float64) / 448.0).astype(np.float32)
    np.testing.assert_array_equal(r["scale_out"], want)
    q = r["quant_out"]
    assert np.all(np.any((q & 0x7F) == 0x7E, axis=1))        # one code at +-448 per row
    assert np.all(q != 0x7F) and np.all(q != 0xFF)              # no NaN codes
    # the codes dequantise to o within half an e4m3 step (relative 2^-4)
    deq = np.vectorize(oracle.e4m3_decode)(q.astype(np.int64)) * r["scale_out"][:, None]
    err = np.abs(deq - r["o"])
    assert np.all(err <= np.abs(r["o"]) * 2.0 ** -4 + r["scale_out"][:, None] * 2.0 ** -10 + 1e-30)


def test_scale_invariance_with_zero_eps():
    """Scaling every partial and the residual by 2^k (exact) leaves o unchanged
    when eps = 0, and scales the new residual by 2^k."""
    inp = random_inputs(4, 16, 256, seed=51)
    ps = [as_u16(p) for p in inp["partials"]]
    res, gam = as_u16(inp["residual"]), as_u16(inp["gamma"])
    base = {p: oracle.fused(ps, res, gam, "bf16", 0.0, 0.0, p, scale_in=0.04) for p in (0, 1, 2)}
    for k in (-3, 5):
        f = 2.0 ** k
        ps2 = [as_u16((inp["partials"][i].double() * f).to(torch.bfloat16)) for i in range(4)]
        res2 = as_u16((inp["residual"].double() * f).to(torch.bfloat16))
        for p in (0, 1, 2):
            s = oracle.fused(ps2, res2, gam, "bf16", 0.0, 0.0, p, scale_in=0.04)
            np.testing.assert_array_equal(base[p]["norm_out"], s["norm_out"])
            if p:
                np.testing.assert_array_equal(base[p]["quant_out"], s["quant_out"])
            np.testing.assert_array_equal(_dec(s["residual_out"], "bf16"),
                                          _dec(base[p]["residual_out"], "bf16") * f)


def test_partial_order_does_not_matter():
    inp = random_inputs(5, 8, 128, seed=61)
    ps = [as_u16(p) for p in inp["partials"]]
    res, gam = as_u16(inp["residual"]), as_u16(inp["gamma"])
    a = oracle.fused(ps, res, gam, "bf16", 1e-6, 0.0, 2)
    b = oracle.fused(ps[::-1], res, gam, "bf16", 1e-6, 0.0, 2)
    for key in ("residual_out", "norm_out", "quant_out", "scale_out"):
        np.testing.assert_array_equal(a[key], b[key])
    # the residual is just one more addend: swapping it with a partial is the same sum
    c = oracle.fused([res] + ps[1:], ps[0], gam, "bf16", 1e-6, 0.0, 2)
    np.testing.assert_array_equal(a["norm_out"], c["norm_out"])


def test_first_pattern_without_residual():
    """No residual input: the new residual is the all-reduce itself."""
    inp = random_inputs(2, 16, 128, seed=71, has_residual=False)
    ps = [as_u16(p) for p in inp["partials"]]
    r = oracle.fused(ps, None, as_u16(inp["gamma"]), "bf16", 1e-6, 0.0, 0, debug=True)
    s = _dec(ps[0], "bf16") + _dec(ps[1], "bf16")
    np.testing.assert_array_equal(r["y"], s)
    np.testing.assert_array_equal(zero_sign_free(r["residual_out"]), zero_sign_free(np_rne16(s, "bf16")))


def test_gamma_is_indexed_by_column():
    """Scaling one column of gamma scales exactly that column of o."""
    inp = random_inputs(2, 4, 64, seed=81)
    ps, res = [as_u16(p) for p in inp["partials"]], as_u16(inp["residual"])
    gam = inp["gamma"].clone()
    a = oracle.fused(ps, res, as_u16(gam), "bf16", 1e-6, 0.0, 0, debug=True)
    gam[5] = gam[5] * 2
    b = oracle.fused(ps, res, as_u16(gam), "bf16", 1e-6, 0.0, 0, debug=True)
    diff = np.nonzero(np.any(a["o"] != b["o"], axis=0))[0].tolist()
    assert diff == [5]
    np.testing.assert_array_equal(b["o"][:, 5], 2 * a["o"][:, 5])


def test_worked_example_fp32_accumulation():
    """The oracle's fp32-accumulation mode (fp32_acc=True taken literally:
    partial 0, 1, ..., then the residual, each addition rounded to fp32)
    against a hand-derived case of rounding followed by cancellation, in
    units of 2^-32: partials -237*2^21, -236, -9*2^24, 129*2^23, residual
    -207*2^21 (bf16 values; their exact sum is -236, i.e. -5.49e-8).
      s1 = -237*2^21                                     (exact)
      s2 = -(237*2^21 + 236) rounds to a multiple of 32 (ulp 2^-27 in
           [2^-4, 2^-3)): 236/32 = 7.375 -> -(237*2^21 + 224)
      s3 = -(309*2^21 + 224) rounds to a multiple of 64 (ulp 2^-26):
           224/64 = 3.5, a tie, to even -> -(309*2^21 + 256)
      s4 = 207*2^21 - 256                                 (exact)
      y  = s4 - 207*2^21 = -256, i.e. -2^-24
    The exact mode keeps -236 * 2^-32: bf16 0xB36C; fp32 accumulation gives
    -2^-24: bf16 0xB380.  The other columns (all partials 1.0, residual 1.0,
    sum 5, exact either way) agree, and so does every output there."""
    units = [-237 * 2 ** 21, -236, -9 * 2 ** 24, 129 * 2 ** 23, -207 * 2 ** 21]
    vals = [u * 2.0 ** -32 for u in units]
    H = 8
    enc = lambda v: oracle.round16(v, "bf16")  # noqa: E731  exact: every value is a bf16
    ps = [np.array([[enc(v)] + [enc(1.0)] * (H - 1)], dtype=np.uint16) for v in vals[:4]]
    res = np.array([[enc(vals[4])] + [enc(1.0)] * (H - 1)], dtype=np.uint16)
    gam = np.array([enc(1.0)] * H, dtype=np.uint16)
    assert [oracle.decode16(int(p[0, 0]), "bf16") for p in ps] == vals[:4]
    ex = oracle.fused(ps, res, gam, "bf16", 1e-6, 0.0, 0)
    f32 = oracle.fused(ps, res, gam, "bf16", 1e-6, 0.0, 0, acc32=True)
    assert ex["residual_out"][0, 0] == 0xB36C
    assert f32["residual_out"][0, 0] == 0xB380
    assert np.array_equal(ex["residual_out"][0, 1:], f32["residual_out"][0, 1:])
    assert oracle.decode16(int(ex["residual_out"][0, 1]), "bf16") == 5.0


@pytest.mark.parametrize("pattern", [0, 1, 2, 3])
def test_fp32_accumulation_equals_exact_without_cancellation(pattern):
    """Where every running fp32 sum is exact the two modes agree bit for bit:
    partials and residual of magnitude in [1, 2) with at most 8 significant
    bits sum exactly in fp32 (sums below 2^6 need at most 14 bits)."""
    rng = np.random.default_rng(11)
    W, T, H = 4, 6, 64
    mags = 1.0 + rng.integers(0, 128, size=(W + 1, T, H)) / 128.0
    signs = np.where(rng.random((W + 1, T, H)) < 0.5, -1.0, 1.0)
    enc = np.vectorize(lambda v: oracle.round16(v, "bf16"))
    arr = enc(mags * signs).astype(np.uint16)
    gam = enc(rng.uniform(0.5, 1.5, H)).astype(np.uint16)
    kw = dict(scale_in=0.05) if pattern == 1 else {}
    ex = oracle.fused(list(arr[:W]), arr[W], gam, "bf16", 1e-6, 0.0, pattern, **kw)
    f32 = oracle.fused(list(arr[:W]), arr[W], gam, "bf16", 1e-6, 0.0, pattern, acc32=True, **kw)
    for k in ("residual_out", "norm_out", "quant_out", "scale_out"):
        if ex.get(k) is not None:
            assert np.array_equal(ex[k], f32[k]), k


def test_golden_small_workload_fixture_is_reproduced():
    """The stored oracle outputs for the small workload (tests/golden) still
    come out of the oracle bit for bit."""
    import os
    import sys
    sys.path.insert(0, os.path.join(os.path.dirname(__file__), "golden"))
    from make_golden import read_fixture
    fx = read_fixture(os.path.join(os.path.dirname(__file__), "golden", "c1_small_oracle.txt"))
    wl = WORKLOADS["c1_small"]
    inp = make_inputs(wl)
    r = oracle.fused([as_u16(p) for p in inp["partials"]], as_u16(inp["residual"]),
                     as_u16(inp["gamma"]), wl.dtype, wl.eps, wl.weight_bias, wl.pattern)
    np.testing.assert_array_equal(r["residual_out"], np.array(fx["residual_out"], np.uint16))
    np.testing.assert_array_equal(r["norm_out"], np.array(fx["norm_out"], np.uint16))
