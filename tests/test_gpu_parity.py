"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Small and ragged shapes are compared element by element; the full-size
workloads (the W=4 8192x8192 static-FP8 prefill and the W=8 4096x7168
per-token-FP8 Gemma workload, the shapes and launch configuration the bench
times) on sampled rows the oracle computes one by one, every outlier row
included.  Tolerances are in gpu_util.
"""
from __future__ import annotations

import json
import os

import numpy as np
import pytest
import torch

from gpu_util import compare, run_gpu, run_oracle, to_gpu
from reduce_residual_add_b200 import far, sp
from reduce_residual_add_b200.inputs import WORKLOADS, make_inputs, random_inputs

pytestmark = pytest.mark.gpu

LOG = os.environ.get("FAR_PARITY_LOG")


def log(name, stats):
    if LOG:
        with open(LOG, "a") as f:
            f.write(json.dumps({"case": name, **{k: v for k, v in stats.items()}}) + "\n")


@pytest.fixture(scope="module")
def ctx():
    c = far.FarContext(0)
    yield c
    c.close()


def _ctx_with_env(env):
    old = {k: os.environ.get(k) for k in env}
    os.environ.update(env)
    try:
        return far.FarContext(0)
    finally:
        for k, v in old.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v


@pytest.fixture(scope="module")
def kctx():
    """Contexts for each prefill kernel: the TMA ring (1 and 2 CTAs per SM)
    and the direct-load kernel."""
    any_rows = {"FAR_RING_MIN_ROWS": "1"}
    out = {"ring": _ctx_with_env(dict(any_rows)),
           # per-tensor FP8: both passes in one ring launch (the
           # default), and in two kernels
           "ring_fused": _ctx_with_env(dict(any_rows, FAR_TENSOR_FUSED="1")),
           "ring_two": _ctx_with_env(dict(any_rows, FAR_TENSOR_FUSED="0")),
           "ring256": _ctx_with_env(dict(any_rows, FAR_RING_THREADS="256", FAR_RING_CTAS_PER_SM="1")),
           "ring3": _ctx_with_env(dict(any_rows, FAR_RING_CTAS_PER_SM="3")),
           "ring2": _ctx_with_env(dict(any_rows, FAR_RING_CTAS_PER_SM="2", FAR_RING_THREADS="256")),
           # gamma read through L1 instead of staged in shared memory
           "ring_l1": _ctx_with_env(dict(any_rows, FAR_RING_GAMMA_SMEM="0")),
           "ring4": _ctx_with_env(dict(any_rows, FAR_RING_CTAS_PER_SM="4", FAR_RING_THREADS="128")),
           "direct": _ctx_with_env({"FAR_PREFILL_KERNEL": "0"})}
    for c in out.values():
        far.far_set_regime(c, far.FAR_REGIME_PREFILL)
    out["decode"] = _ctx_with_env({})
    far.far_set_regime(out["decode"], far.FAR_REGIME_DECODE)
    yield out
    for c in out.values():
        c.close()


@pytest.fixture
def regime(ctx):
    """Set a regime for one test and restore automatic choice afterwards."""
    def set_(r):
        far.far_set_regime(ctx, r)
    yield set_
    far.far_set_regime(ctx, far.FAR_REGIME_AUTO)


# (W, T, H, dtype, pattern, has_residual, weight_bias)
SMALL = [
    (2, 8, 64, "bf16", 0, True, 0.0),       # the small workload's shape
    (1, 5, 8, "bf16", 0, True, 0.0),        # one pack per row
    (3, 37, 256, "fp16", 1, True, 0.0),     # 32 packs: rows inside a warp
    (4, 33, 264, "bf16", 2, True, 1.0),     # 33 packs: a ragged second warp
    (5, 17, 1000, "bf16", 1, False, 0.0),   # ragged H, no residual
    (8, 40, 4096, "bf16", 0, True, 0.0),
    (16, 9, 2048, "fp16", 2, True, 0.0),    # the largest W
    (2, 130, 7168, "bf16", 2, True, 1.0),
    (4, 70, 8192, "bf16", 1, True, 0.0),
    (3, 11, 8200, "fp16", 0, True, 0.0),    # 1025 packs: 8 per thread, ragged
    (2, 6, 16384, "bf16", 2, True, 0.0),    # the largest H
    (1, 64, 512, "bf16", 2, True, 0.0),     # one rank: plain add + RMSNorm
    (7, 3, 6144, "fp16", 1, True, 1.0),
]


@pytest.mark.parametrize("reg", [far.FAR_REGIME_AUTO, far.FAR_REGIME_DECODE, far.FAR_REGIME_PREFILL])
@pytest.mark.parametrize("case", SMALL, ids=lambda c: "W%d_T%d_H%d_%s_p%d_res%d_wb%g" % c)
def test_small_shapes(ctx, regime, case, reg):
    W, T, H, dt, pattern, has_res, wb = case
    regime(reg)
    inp = random_inputs(W, T, H, dtype=dt, seed=W * 1000 + T * 7 + H, has_residual=has_res)
    eps, scale = 1e-6, 0.05
    got = run_gpu(ctx, to_gpu(inp), eps, wb, pattern, scale_in=scale, guard=4096)
    ref = run_oracle(inp, dt, eps, wb, pattern, scale_in=scale)
    log("small %s reg%d" % (case, reg), compare(got, ref, dt))


@pytest.mark.parametrize("kern", ["ring", "ring256", "ring3", "ring2", "ring_l1", "ring4", "direct"])
@pytest.mark.parametrize("case", [
    (2, 3000, 264, "bf16", 2, True, 0.0),    # 33 packs, 32 slots, ~20 rows per CTA
    (16, 300, 16384, "bf16", 1, True, 1.0),  # 17 segments per row, 6 slots
    (4, 1000, 8192, "fp16", 0, False, 0.0),  # no residual: W segments per row
    (8, 149, 7168, "bf16", 2, True, 1.0),    # one more row than CTAs
    (3, 7, 2048, "bf16", 1, True, 0.0),      # fewer rows than CTAs
    (2, 1200, 12288, "bf16", 1, True, 0.0),  # 1536 packs: the wide build (384 consumers)
    (8, 300, 10248, "fp16", 2, True, 1.0),   # 1281 packs, ragged: wide, 352 consumers
], ids=lambda c: "W%d_T%d_H%d_%s_p%d_res%d_wb%g" % c)
def test_prefill_kernels(kctx, case, kern):
    W, T, H, dt, pattern, has_res, wb = case
    c = kctx[kern]
    info = far.far_describe_launch(c, T, H, torch.bfloat16, W, has_res)
    per_sm = {"ring4": 4, "ring3": 3, "ring2": 2}.get(kern, 1)
    fits = 228 * 1024 // per_sm - 1024 >= 3 * H * 2 + 1024   # gamma, two slots, header
    assert info["kernel"] == (1 if (kern != "direct" and fits) else 0)
    inp = random_inputs(W, T, H, dtype=dt, seed=7 * W + T + H, has_residual=has_res)
    got = run_gpu(c, to_gpu(inp), 1e-6, wb, pattern, scale_in=0.05, guard=1024)
    ref = run_oracle(inp, dt, 1e-6, wb, pattern, scale_in=0.05)
    log("prefill %s %s" % (kern, case), compare(got, ref, dt))


@pytest.mark.parametrize("case", [
    (2, 1200, 12288, "bf16", 1, 0.0),   # 1536 packs: 384 consumers
    (3, 700, 10248, "fp16", 2, 1.0),    # 1281 packs, ragged: 352 consumers
    (2, 600, 16384, "bf16", 1, 0.0),    # 2048 packs: one CTA of 512 consumers
    (3, 400, 14344, "fp16", 2, 1.0),    # 1793 packs, ragged: 480 consumers
], ids=lambda c: "W%d_T%d_H%d_%s_p%d_wb%g" % c)
def test_ring_wide_build(kctx, case):
    """Rows of 1025-2048 packs without norm_out take a wide build (4 packs
    per thread over up to 384 or 512 consumers)."""
    W, T, H, dt, pattern, wb = case
    c = kctx["ring"]
    info = far.far_describe_launch(c, T, H, torch.bfloat16, W, True, False)
    assert (info["kernel"], info["packs_per_thread"]) == (1, 4)
    assert info["threads_per_cta"] == ((H // 8 + 3) // 4 + 31) // 32 * 32 + 32
    inp = random_inputs(W, T, H, dtype=dt, seed=11 * W + T + H, has_residual=True)
    got = run_gpu(c, to_gpu(inp), 1e-6, wb, pattern, scale_in=0.05, guard=1024, want_norm=False)
    ref = run_oracle(inp, dt, 1e-6, wb, pattern, scale_in=0.05, want_norm=False)
    log("ring wide %s" % (case,), compare(got, ref, dt))


@pytest.mark.parametrize("pattern", [1, 2])
def test_ring_and_direct_agree_bitwise(kctx, pattern):
    """With the same threads per row, both prefill kernels sum in the same
    order and reduce in the same tree: identical bits."""
    inp = random_inputs(4, 600, 8192, seed=21)
    g = to_gpu(inp)
    a = run_gpu(kctx["ring256"], g, 1e-5, 0.0, pattern, scale_in=0.05)
    b = run_gpu(kctx["direct"], g, 1e-5, 0.0, pattern, scale_in=0.05)
    c = run_gpu(kctx["ring2"], g, 1e-5, 0.0, pattern, scale_in=0.05)
    for k in ("residual_out", "norm_out", "quant_out", "scale_out"):
        if a[k] is not None:
            assert np.array_equal(a[k], b[k]) and np.array_equal(a[k], c[k]), k


def test_small_workload_matches_golden_fixture(ctx):
    import sys
    sys.path.insert(0, os.path.join(os.path.dirname(__file__), "golden"))
    from make_golden import read_fixture
    fx = read_fixture(os.path.join(os.path.dirname(__file__), "golden", "c1_small_oracle.txt"))
    wl = WORKLOADS["c1_small"]
    inp = make_inputs(wl)
    got = run_gpu(ctx, to_gpu(inp), wl.eps, wl.weight_bias, wl.pattern)
    ref = {"residual_out": np.array(fx["residual_out"], np.uint16),
           "norm_out": np.array(fx["norm_out"], np.uint16)}
    log("c1 golden", compare(got, ref, "bf16"))


@pytest.mark.parametrize("T", [1, 8, 32, 80])
@pytest.mark.parametrize("reg", [far.FAR_REGIME_AUTO, far.FAR_REGIME_DECODE, far.FAR_REGIME_PREFILL])
def test_decode_workload(ctx, regime, T, reg):
    wl = WORKLOADS["c2_decode_T%d" % T]
    regime(reg)
    info = far.far_describe_launch(ctx, T, wl.H, torch.bfloat16, wl.W, True)
    if reg == far.FAR_REGIME_DECODE:
        assert info["regime"] == far.FAR_REGIME_DECODE and info["ctas_per_row"] >= 2
    inp = make_inputs(wl)
    got = run_gpu(ctx, to_gpu(inp), wl.eps, wl.weight_bias, wl.pattern, guard=256)
    ref = run_oracle(inp, wl.dtype, wl.eps, wl.weight_bias, wl.pattern)
    log("c2 T%d reg%d" % (T, reg), compare(got, ref, wl.dtype))


def test_3d_input_and_row_slices(ctx):
    """[4, 256, 2048] tensors go in as they are (the binding takes the 2-D
    view); two 512-row slices equal the full call bit for bit."""
    wl = WORKLOADS["c3_3d"]
    inp = make_inputs(wl)
    g = to_gpu(inp)
    g3 = {"partials": [p.view(4, 256, 2048) for p in g["partials"]],
          "residual": g["residual"].view(4, 256, 2048), "gamma": g["gamma"]}
    full = run_gpu(ctx, g3, wl.eps, 0.0, 0)
    ref = run_oracle(inp, "bf16", wl.eps, 0.0, 0)
    log("c3 full", compare(full, ref, "bf16"))
    for pattern in (0, 1, 2):
        whole = run_gpu(ctx, g, wl.eps, 0.0, pattern, scale_in=0.05)
        ps = g["partials"]
        T, H = 1024, 2048
        rout = torch.zeros(T, H, dtype=torch.bfloat16, device="cuda")
        nout = torch.zeros_like(rout)
        qout = torch.zeros(T, H, dtype=torch.uint8, device="cuda") if pattern else None
        sout = torch.zeros(T, dtype=torch.float32, device="cuda") if pattern == 2 else None
        sin = torch.tensor([0.05], device="cuda") if pattern == 1 else None
        for b, e in ((0, 512), (512, 1024)):
            far.far_fused_rows(ctx, b, e, ps, g["residual"], g["gamma"], wl.eps, 0.0, pattern,
                               residual_out=rout, norm_out=nout, quant_out=qout, scale_in=sin,
                               scale_out=sout)
        torch.cuda.synchronize()
        from reduce_residual_add_b200.inputs import as_u16
        assert np.array_equal(as_u16(rout.cpu()), whole["residual_out"])
        assert np.array_equal(as_u16(nout.cpu()), whole["norm_out"])
        if pattern:
            assert np.array_equal(qout.cpu().numpy(), whole["quant_out"])
        if pattern == 2:
            assert np.array_equal(sout.cpu().numpy(), whole["scale_out"])


@pytest.mark.parametrize("G,T,H,pattern", [(2, 1024, 2048, 0), (4, 4096, 8192, 1), (8, 640, 4096, 2)])
def test_sequence_parallel_local_steps_equal_the_full_call(ctx, G, T, H, pattern):
    """The kernel side of the sequence-parallel path (reduce_residual_add_b200.sp),
    each rank's step run in turn on this GPU: rank r's local call gets the
    G partial blocks of its rows as G separate buffers (what the row exchange
    delivers) and its rows of the residual; stitched together, the outputs
    equal the one-call result over all T rows bit for bit."""
    inp = random_inputs(G, T, H, seed=700 + G)
    g = to_gpu(inp)
    scale = 0.05
    whole = run_gpu(ctx, g, 1e-6, 0.0, pattern, scale_in=scale, want_norm=pattern == 0)
    n = T // G
    parts = {k: [] for k in ("residual_out", "norm_out", "quant_out", "scale_out")}
    for r in range(G):
        b, e = sp.rows_for_rank(T, G, r)
        recv = [p_[b:e].clone() for p_ in g["partials"]]     # block j from rank j
        local = {"partials": recv, "residual": g["residual"][b:e].clone(), "gamma": g["gamma"]}
        got = run_gpu(ctx, local, 1e-6, 0.0, pattern, scale_in=scale, want_norm=pattern == 0)
        for k in parts:
            if got[k] is not None:
                parts[k].append(got[k])
    for k, v in parts.items():
        if whole[k] is None:
            continue
        assert np.array_equal(np.concatenate(v), whole[k]), k
    assert n * G == T
    compare(whole, run_oracle(inp, "bf16", 1e-6, 0.0, pattern, scale_in=scale,
                              want_norm=pattern == 0), "bf16")


def test_row_slices_leave_other_rows_alone(ctx):
    inp = random_inputs(3, 100, 1024, seed=5)
    g = to_gpu(inp)
    got = run_gpu(ctx, g, 1e-6, 0.0, 2, rows=(17, 61))
    ref = run_oracle(inp, "bf16", 1e-6, 0.0, 2, rows=(17, 61))
    log("rows 17..61", compare(got, ref, "bf16"))
    # untouched rows keep the zeros run_gpu put there
    for key in ("residual_out", "norm_out", "quant_out"):
        assert not got[key][:17].any() and not got[key][61:].any()
    assert not got["scale_out"][:17].any() and not got["scale_out"][61:].any()


def _sample_rows(T, outliers, n, seed):
    g = np.random.default_rng(seed)
    rows = set(g.choice(T, size=n, replace=False).tolist())
    rows |= {0, 1, T - 2, T - 1}
    rows |= set(int(r) for r in outliers)
    return np.array(sorted(rows))


@pytest.mark.parametrize("with_norm", [False, True])
def test_prefill_static_fp8_full_size(ctx, with_norm):
    wl = WORKLOADS["c4_prefill_fp8_static"]
    inp = make_inputs(wl)
    g = to_gpu(inp)
    got = run_gpu(ctx, g, wl.eps, wl.weight_bias, wl.pattern, scale_in=wl.static_scale,
                  want_norm=with_norm)
    rows = _sample_rows(wl.T, inp["outlier_rows"].tolist(), 160, 3)
    ref = run_oracle(inp, wl.dtype, wl.eps, wl.weight_bias, wl.pattern,
                     scale_in=wl.static_scale, want_norm=with_norm, row_list=rows)
    log("c4 norm=%s" % with_norm, compare(got, ref, wl.dtype, rows=rows))


@pytest.mark.parametrize("dt", ["bf16", "fp16"])
def test_gemma_token_fp8_full_size(ctx, dt):
    wl = WORKLOADS["c5_gemma_fp8_token_%s" % dt]
    inp = make_inputs(wl)
    got = run_gpu(ctx, to_gpu(inp), wl.eps, wl.weight_bias, wl.pattern)
    rows = _sample_rows(wl.T, [], 160, 4)
    ref = run_oracle(inp, dt, wl.eps, wl.weight_bias, wl.pattern, row_list=rows)
    log("c5 %s" % dt, compare(got, ref, dt, rows=rows))
    # properties at every row: one code at +-448 per row, scale > 0
    q = got["quant_out"]
    assert np.all(np.any((q & 0x7F) == 0x7E, axis=1))
    assert np.all(got["scale_out"] > 0)


def test_deterministic(ctx):
    inp = random_inputs(4, 300, 7168, seed=9)
    g = to_gpu(inp)
    a = run_gpu(ctx, g, 1e-6, 1.0, 2)
    b = run_gpu(ctx, g, 1e-6, 1.0, 2)
    for k in ("residual_out", "norm_out", "quant_out", "scale_out"):
        assert np.array_equal(a[k], b[k]), k


def test_in_place_residual_and_side_stream(ctx):
    inp = random_inputs(2, 50, 2048, seed=10)
    s = torch.cuda.Stream()
    got = run_gpu(ctx, to_gpu(inp), 1e-6, 0.0, 1, scale_in=0.1, in_place=True, stream=s)
    ref = run_oracle(inp, "bf16", 1e-6, 0.0, 1, scale_in=0.1)
    log("in place", compare(got, ref, "bf16"))


def test_first_pattern_without_residual(ctx, regime):
    for reg in (far.FAR_REGIME_DECODE, far.FAR_REGIME_PREFILL):
        regime(reg)
        inp = random_inputs(4, 12, 4096, seed=11, has_residual=False)
        got = run_gpu(ctx, to_gpu(inp), 1e-6, 0.0, 2)
        ref = run_oracle(inp, "bf16", 1e-6, 0.0, 2)
        compare(got, ref, "bf16")
        # norm only: no residual in, no residual out
        got = run_gpu(ctx, to_gpu(inp), 1e-6, 0.0, 0, want_residual_out=False)
        ref = run_oracle(inp, "bf16", 1e-6, 0.0, 0, want_residual_out=False)
        compare(got, ref, "bf16")


def test_zero_rows_saturation_and_nonfinite(ctx):
    inp = random_inputs(2, 6, 1024, seed=12)
    inp["partials"][0][1].zero_()
    inp["partials"][1][1].zero_()
    inp["residual"][1].zero_()                        # row 1 is all zero
    inp["partials"][0][3, 5] = float("inf")           # row 3: inf -> NaN row
    inp["partials"][1][4, 7] = float("nan")           # row 4: NaN row
    for pattern, scale in ((0, None), (1, 2.0 ** -12), (2, None)):
        got = run_gpu(ctx, to_gpu(inp), 1e-6, 0.0, pattern, scale_in=scale)
        ref = run_oracle(inp, "bf16", 1e-6, 0.0, pattern, scale_in=scale)
        compare(got, ref, "bf16")
        if pattern == 1:
            assert np.all(got["quant_out"][0][(ref["quant_out"][0] & 0x7F) == 0x7E] & 0x7F == 0x7E)
        if pattern == 2:
            # the zero row and the rows with an inf / a NaN input: scale 0, codes 0
            for r in (1, 3, 4):
                assert got["scale_out"][r] == 0 and not got["quant_out"][r].any()


def test_empty_problem_and_slice_are_noops(ctx):
    inp = random_inputs(2, 4, 64, seed=13)
    g = to_gpu(inp)
    rout = torch.full((4, 64), 7, dtype=torch.bfloat16, device="cuda")
    nout = torch.full_like(rout, 7)
    far.far_fused_rows(ctx, 2, 2, g["partials"], g["residual"], g["gamma"], 1e-6, 0.0, 0,
                       residual_out=rout, norm_out=nout)
    e = [torch.empty(0, 64, dtype=torch.bfloat16, device="cuda")] * 2
    far.far_fused(ctx, e, e[0], g["gamma"], 1e-6, 0.0, 0, residual_out=e[0].clone(),
                  norm_out=e[0].clone())
    torch.cuda.synchronize()
    assert bool((rout == 7).all()) and bool((nout == 7).all())


def test_errors_are_reported_not_skipped(ctx):
    inp = random_inputs(2, 4, 64, seed=14)
    g = to_gpu(inp)
    out = torch.empty(4, 64, dtype=torch.bfloat16, device="cuda")
    bad = torch.empty(4 * 64 + 8, dtype=torch.bfloat16, device="cuda")[1:1 + 4 * 64].view(4, 64)
    with pytest.raises(far.FarError) as e:
        far.far_fused(ctx, g["partials"], g["residual"], g["gamma"], 1e-6, 0.0, 0,
                      residual_out=out, norm_out=bad)
    assert e.value.status == far.FAR_ERR_ALIGNMENT
    with pytest.raises(far.FarError) as e:
        far.far_fused(ctx, g["partials"], g["residual"], g["gamma"], 1e-6, 0.0, 0, residual_out=out)
    assert e.value.status == far.FAR_ERR_INVALID_ARG
    with pytest.raises(far.FarError) as e:
        far.far_fused(ctx, g["partials"], g["residual"], g["gamma"], 1e-6, 0.0, 0,
                      residual_out=out, norm_out=g["partials"][0])
    assert e.value.status == far.FAR_ERR_INVALID_ARG
    p12 = [torch.zeros(2, 12, dtype=torch.bfloat16, device="cuda")]
    with pytest.raises(far.FarError) as e:
        far.far_fused(ctx, p12, None, torch.ones(12, dtype=torch.bfloat16, device="cuda"), 1e-6,
                      0.0, 0, norm_out=torch.empty(2, 12, dtype=torch.bfloat16, device="cuda"))
    assert e.value.status == far.FAR_ERR_UNSUPPORTED


def test_launch_plan(ctx):
    """The measured dispatch rules (see far_abi.cu plan())."""
    d = lambda rows, H, W, res=True, norm=False: far.far_describe_launch(  # noqa: E731
        ctx, rows, H, torch.bfloat16, W, res, norm)
    # decode-sized rows: a cluster per row once one CTA would need 4 packs
    # per thread (H >= 8192), 16 CTAs per row up to 4 rows, 8 up to 16, else 4 ...
    cl = lambda rows, H, W: (d(rows, H, W)["regime"], d(rows, H, W)["ctas_per_row"])  # noqa: E731
    assert cl(4, 16384, 8) == (far.FAR_REGIME_DECODE, 16)
    assert cl(1, 8192, 8) == (far.FAR_REGIME_DECODE, 16)
    assert cl(1, 8192, 2) == (far.FAR_REGIME_DECODE, 16)
    assert cl(8, 8192, 2) == (far.FAR_REGIME_DECODE, 8)
    assert cl(64, 8192, 8) == (far.FAR_REGIME_DECODE, 4)
    # ... halved while the grid would not be resident in one wave
    assert cl(80, 16384, 2) == (far.FAR_REGIME_DECODE, 2)
    # ... one CTA per row for smaller ones (W=8, H=4096: 2 packs per thread)
    assert d(80, 4096, 8)["regime"] == far.FAR_REGIME_PREFILL
    assert d(1, 4096, 2)["regime"] == far.FAR_REGIME_PREFILL
    assert d(81, 16384, 8)["regime"] == far.FAR_REGIME_PREFILL
    # below the ring threshold the threads per row do not depend on the rows
    # (row slices reduce in the same order as the whole call)
    c3 = d(1024, 2048, 2)
    assert (c3["kernel"], c3["threads_per_cta"], c3["packs_per_thread"]) == (0, 256, 1)
    assert d(256, 2048, 2)["threads_per_cta"] == 256
    # prefill: the ring from ~8 rows per persistent CTA, the direct kernel below
    c4 = d(8192, 8192, 4)
    assert c4["kernel"] == 1 and c4["ring_slots"] >= 2
    assert (c4["threads_per_cta"] - 32) * c4["packs_per_thread"] * 8 >= 8192
    assert d(1200, 8192, 4)["kernel"] == 0
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    # 5-6 segments of 1024 packs: 3 CTAs per SM x 3 slots, gamma in shared memory
    assert (c4["grid_ctas"], c4["ring_gamma_smem"], c4["ring_slots"]) == (3 * sms, 1, 3)
    # ... 3 segments: 2 CTAs per SM x 4 slots
    w2 = d(8192, 8192, 2)
    assert (w2["grid_ctas"], w2["ring_gamma_smem"], w2["ring_slots"]) == (2 * sms, 1, 4)
    # ... but with norm_out, 2 CTAs per SM, gamma through L1, ~96 KiB of slots
    c4n = d(8192, 8192, 4, norm=True)
    assert (c4n["grid_ctas"], c4n["ring_gamma_smem"], c4n["ring_slots"]) == (2 * sms, 0, 6)
    # 8 or more segments of 513-896 packs: the wide 2-pack build (448
    # consumers), 2 CTAs per SM x 4 slots, gamma in shared memory
    c5 = d(4096, 7168, 8)
    assert (c5["grid_ctas"], c5["ring_gamma_smem"], c5["ring_slots"]) == (2 * sms, 1, 4)
    assert (c5["packs_per_thread"], c5["threads_per_cta"]) == (2, 480)
    assert d(4096, 7168, 4)["packs_per_thread"] == 4
    # rows of at most 384 packs: 4 CTAs per SM x 4 slots, whatever the segments
    h3 = d(32768, 3072, 8)
    assert (h3["grid_ctas"], h3["ring_slots"]) == (4 * sms, 4)
    # H=4096 with few segments: 4 packs per thread (128 consumers), and
    # without norm_out 4 CTAs per SM x 3 slots (3 CTAs with it)
    h4 = d(16384, 4096, 4)
    assert (h4["packs_per_thread"], h4["threads_per_cta"], h4["grid_ctas"], h4["ring_slots"]) == (4, 160, 4 * sms, 3)
    assert d(16384, 4096, 4, norm=True)["grid_ctas"] == 3 * sms
    # 1025-1536 packs without norm_out: the wide build, 4 packs per thread
    h12 = d(8192, 12288, 2)
    assert (h12["packs_per_thread"], h12["threads_per_cta"], h12["grid_ctas"], h12["ring_slots"]) == (4, 416, 2 * sms, 3)
    # ... with norm_out and at most 6 segments, gamma through L1 and 2 slots
    h12n = d(8192, 12288, 2, norm=True)
    assert (h12n["packs_per_thread"], h12n["ring_gamma_smem"], h12n["ring_slots"]) == (4, 0, 2)
    # 1537-2048 packs without norm_out: one CTA per SM of 512 consumers, 4
    # slots for at most 4 segments (6 beyond)
    h16 = d(8192, 16384, 2)
    assert (h16["kernel"], h16["grid_ctas"], h16["ring_gamma_smem"], h16["ring_slots"]) == (1, sms, 1, 4)
    assert d(8192, 16384, 4)["ring_slots"] == 6
    assert (h16["packs_per_thread"], h16["threads_per_cta"]) == (4, 544)
    # ... with norm_out and at most 6 segments: 8 packs per thread, 2 CTAs
    # per SM, gamma in shared memory
    h16n = d(8192, 16384, 2, norm=True)
    assert (h16n["packs_per_thread"], h16n["grid_ctas"], h16n["ring_slots"]) == (8, 2 * sms, 2)
    # ... with more segments, the one-CTA build with 6 slots
    h16w8 = d(8192, 16384, 8, norm=True)
    assert (h16w8["grid_ctas"], h16w8["ring_gamma_smem"], h16w8["ring_slots"]) == (sms, 1, 6)
    # rows of at most 256 packs: 128 consumers, 6 CTAs per SM x 4 slots
    # (4 x 6 with norm_out)
    h2 = d(32768, 2048, 4)
    assert (h2["threads_per_cta"], h2["packs_per_thread"], h2["grid_ctas"], h2["ring_slots"]) == (160, 2, 6 * sms, 4)
    h2n = d(32768, 2048, 4, norm=True)
    assert (h2n["grid_ctas"], h2n["ring_slots"]) == (4 * sms, 6)
    # 768 packs: 4 CTAs per SM x 2 slots; with norm_out 2 x 4
    h6 = d(8192, 6144, 4, norm=True)
    assert (h6["grid_ctas"], h6["ring_gamma_smem"], h6["ring_slots"]) == (2 * sms, 1, 4)
    h6p = d(8192, 6144, 4)
    assert (h6p["grid_ctas"], h6p["ring_slots"]) == (4 * sms, 2)
    tiny = d(8, 64, 2)
    assert tiny["regime"] == far.FAR_REGIME_PREFILL and tiny["rows_per_cta"] > 1


def test_launch_plan_tensor_and_group(ctx):
    """Per-tensor and per-group FP8 plan the ring kernel by rules of their
    own (see far_abi.cu plan_ring) and never take the cluster kernel."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count

    def d(rows, H, W, pattern, norm=False):
        return far.far_describe_launch(ctx, rows, H, torch.bfloat16, W, True, norm, pattern=pattern)

    def geo(i):
        return (i["kernel"], i["grid_ctas"], i["ring_slots"])

    T3, G4 = far.FAR_AR_RESIDUAL_RMSNORM_FP8_TENSOR, far.FAR_AR_RESIDUAL_RMSNORM_FP8_GROUP
    # patterns 0-2 share far_describe_launch's plan
    for pat in (0, 1, 2):
        assert d(8192, 8192, 4, pat) == far.far_describe_launch(ctx, 8192, 8192, torch.bfloat16, 4, True)
    # per-tensor, H <= 2048: 6 CTAs per SM x 4 slots, with norm_out too
    # (the static rule: 4 x 6 with norm_out)
    assert geo(d(32768, 2048, 2, T3)) == (1, 6 * sms, 4)
    assert geo(d(32768, 2048, 4, T3, norm=True)) == (1, 6 * sms, 4)
    # ... H = 3072 with norm_out: 4 x 6 (static: 3 x 4)
    h3 = d(32768, 3072, 4, T3, norm=True)
    assert (geo(h3), h3["threads_per_cta"]) == ((1, 4 * sms, 6), 224)
    assert geo(d(32768, 3072, 4, None, norm=True)) == (1, 3 * sms, 4)
    # ... H = 4096, at most 6 segments: 5 x 4 (static: 4 x 3)
    h4 = d(16384, 4096, 4, T3)
    assert (geo(h4), h4["packs_per_thread"]) == ((1, 5 * sms, 4), 4)
    # ... H = 8192: 3 x 3 for every W (static at W=2: 2 x 4)
    assert geo(d(8192, 8192, 2, T3)) == (1, 3 * sms, 3)
    assert geo(d(8192, 8192, 4, T3)) == (1, 3 * sms, 3)
    assert geo(d(8192, 8192, 2, None)) == (1, 2 * sms, 4)
    # per-group, up to 256 packs and 6 segments: 5 x 6
    assert geo(d(32768, 2048, 2, G4)) == (1, 5 * sms, 6)
    # decode-sized calls of both stay on one CTA per row
    assert d(4, 16384, 8, None)["regime"] == far.FAR_REGIME_DECODE
    for pat in (T3, G4):
        i = d(4, 16384, 8, pat)
        assert (i["regime"], i["ctas_per_row"], i["grid_ctas"]) == (far.FAR_REGIME_PREFILL, 1, 4)
    with pytest.raises(far.FarError) as e:
        d(8192, 8192, 4, 5)
    assert e.value.status == far.FAR_ERR_INVALID_ARG


@pytest.mark.parametrize("kern", ["decode", "ring", "direct"])
def test_chained_calls_read_completed_outputs(kctx, ctx, kern):
    """With programmatic dependent launch each call must still read what the
    previous call wrote: call k+1 takes call k's new residual as its
    residual, four times in a stream and four times inside a CUDA graph."""
    H, W = 4096, 4
    T = 4 if kern == "decode" else 600
    c = kctx[kern]
    inps = [random_inputs(W, T, H, seed=300 + k) for k in range(4)]
    g = [to_gpu(i) for i in inps]
    gam = g[0]["gamma"]
    res0 = g[0]["residual"]

    def chain(stream):
        outs = []
        res = res0
        for k in range(4):
            rout = torch.empty_like(res0)
            nout = torch.empty_like(res0)
            far.far_fused(c, g[k]["partials"], res, gam, 1e-6, 0.0, 0,
                          residual_out=rout, norm_out=nout, stream=stream)
            outs.append((rout, nout))
            res = rout
        return outs

    s = torch.cuda.Stream()
    outs = chain(s)
    torch.cuda.synchronize()
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gr, stream=s):
        gouts = chain(s)
    with torch.cuda.stream(s):
        gr.replay()
    torch.cuda.synchronize()
    far.far_check(c)
    info = far.far_describe_launch(c, T, H, torch.bfloat16, W, True)
    assert (info["regime"], info["kernel"]) == {"decode": (1, 0), "ring": (2, 1), "direct": (2, 0)}[kern]
    from reduce_residual_add_b200.inputs import as_u16
    import oracle
    gam16 = as_u16(inps[0]["gamma"].contiguous())
    for run in (outs, gouts):
        prev = as_u16(inps[0]["residual"])
        for k in range(4):
            ref = oracle.fused([as_u16(p) for p in inps[k]["partials"]], prev, gam16, "bf16",
                               1e-6, 0.0, 0)
            got_r = as_u16(run[k][0].cpu())
            got_n = as_u16(run[k][1].cpu())
            assert compare({"residual_out": got_r, "norm_out": got_n}, ref, "bf16") is not None
            prev = got_r          # the next call reads exactly what this one wrote
    del gr



# ---------------------------------------------------------------------------
# dynamic per-tensor FP8 (two passes, workspace)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("norm", [True, False], ids=["norm_out", "codes_from_new_residual"])
@pytest.mark.parametrize("kern", ["ring_fused", "ring_two", "direct", "auto"])
@pytest.mark.parametrize("case", [
    (2, 8, 64, "bf16", True, 0.0),
    (8, 5, 4096, "bf16", True, 0.0),        # decode-sized: never the cluster kernel
    (4, 300, 8192, "fp16", True, 1.0),
    (3, 1000, 1000, "bf16", False, 0.0),
    (16, 40, 16384, "bf16", True, 0.0),
    (2, 77, 8200, "bf16", True, 0.0),      # 1025 packs: 8 per thread, ragged
    (8, 300, 5128, "bf16", True, 0.0),     # 641 packs, 9 segments: the 448-consumer build
], ids=lambda c: "W%d_T%d_H%d_%s_res%d_wb%g" % c)
def test_per_tensor_fp8(kctx, ctx, case, kern, norm):
    """The second pass forms the codes from what the first pass stored:
    norm_out (rounded o) when the call writes it, else the new residual
    (rounded y); codes within one step of the oracle's, saturation included,
    and the scale from the unrounded o."""
    W, T, H, dt, has_res, wb = case
    c = ctx if kern == "auto" else kctx[kern]
    inp = random_inputs(W, T, H, dtype=dt, seed=500 + W + T + H, has_residual=has_res)
    got = run_gpu(c, to_gpu(inp), 1e-6, wb, 3, guard=512, want_norm=norm)
    ref = run_oracle(inp, dt, 1e-6, wb, 3, want_norm=norm)
    st = compare(got, ref, dt, exact_saturation=False)
    log("tensor %s %s norm=%d" % (kern, case, norm), st)
    assert np.any((got["quant_out"] & 0x7F) == 0x7E)
    assert st["quant_out"][1] > 0.95                            # most codes exact


@pytest.mark.parametrize("norm", [False, True])
@pytest.mark.parametrize("kern", ["ring_fused", "ring_two", "auto"])
@pytest.mark.parametrize("in_place", [False, True])
def test_per_tensor_fp8_rebuilt_rows(kctx, ctx, in_place, kern, norm):
    """Codes from the stored new residual or norm_out: rows that may overflow
    the format (fp16 sums past 65504, whose new residual is +inf) and rows
    with an inf or NaN input are flagged by the first pass, which stores no
    new residual for them; the second pass rebuilds their y from the
    inputs, in place too (the residual is still intact).  "ring_fused":
    both passes in one launch; "ring_two", "auto" (300 rows: the one-CTA
    kernel): two kernels."""
    c = ctx if kern == "auto" else kctx[kern]
    T, H = 300, 4096
    inp = random_inputs(4, T, H, dtype="fp16", seed=93)
    for p_ in inp["partials"]:
        p_[::7, :16] = 30000.0
    inp["partials"][0][5, 9] = float("inf")
    inp["partials"][1][6, 3] = float("nan")
    got = run_gpu(c, to_gpu(inp), 1e-6, 0.0, 3, want_norm=norm, in_place=in_place)
    ref = run_oracle(inp, "fp16", 1e-6, 0.0, 3, want_norm=norm)
    compare(got, ref, "fp16", exact_saturation=False)
    assert np.all(got["residual_out"][::7, :16] == 0x7C00)          # +inf


@pytest.mark.parametrize("kern", ["ring_fused", "ring_two", "auto"])
def test_per_tensor_fp8_norm_out_past_the_format(kctx, ctx, kern):
    """Codes from the stored norm_out: a row with an element of o past the
    format's largest finite value (infinite in norm_out, as in the oracle)
    is flagged by the first pass and its codes are formed from o itself."""
    c = ctx if kern == "auto" else kctx[kern]
    T, H = 300, 2048
    inp = random_inputs(2, T, H, dtype="fp16", seed=95)
    inp["gamma"][[7, 100, 901, 2000]] = 40000.0
    got = run_gpu(c, to_gpu(inp), 1e-6, 0.0, 3, want_norm=True)
    ref = run_oracle(inp, "fp16", 1e-6, 0.0, 3, want_norm=True)
    compare(got, ref, "fp16", exact_saturation=False)
    infs = (ref["norm_out"] & 0x7FFF) == 0x7C00
    assert infs.any(axis=1).sum() > 10 and (~infs.any(axis=1)).sum() > 10


def test_per_tensor_fp8_without_residual_output(ctx):
    """No residual in and no new residual out: nothing to read back, so the
    second pass reads the inputs again; with a residual_out it reads that."""
    inp = random_inputs(3, 200, 2048, seed=94, has_residual=False)
    for want_rout in (False, True):
        got = run_gpu(ctx, to_gpu(inp), 1e-6, 0.0, 3, want_norm=False,
                      want_residual_out=want_rout)
        ref = run_oracle(inp, "bf16", 1e-6, 0.0, 3, want_norm=False,
                         want_residual_out=want_rout)
        compare(got, ref, "bf16", exact_saturation=False)
    

def test_per_tensor_fp8_full_size_c4_shape(ctx):
    """The c4 prefill shape (W=4, 8192 x 8192 bf16, 82 outlier rows x50) with
    dynamic per-tensor FP8 and no norm_out, as the bench times it: every row
    against the oracle (the scale spans all rows)."""
    wl = WORKLOADS["c4_prefill_fp8_tensor"]
    inp = make_inputs(wl)
    got = run_gpu(ctx, to_gpu(inp), wl.eps, wl.weight_bias, 3, want_norm=False)
    ref = run_oracle(inp, "bf16", wl.eps, wl.weight_bias, 3, want_norm=False)
    st = compare(got, ref, "bf16", exact_saturation=False)
    log("tensor c4 full", st)
    assert st["quant_out"][1] > 0.95


@pytest.mark.parametrize("case", [
    (2, 77, 64, "direct"),      # several rows per CTA, a partly filled last CTA
    (4, 600, 8192, "ring"),     # persistent CTAs, more rows than CTAs
    (8, 9, 4096, "auto"),       # decode-sized
], ids=lambda c: "W%d_T%d_H%d_%s" % c)
def test_per_tensor_fp8_row_order(case):
    """The second pass may take the rows last row first: every output is the
    same bit for bit (each row's arithmetic is untouched, the scale is a max)."""
    W, T, H, kern = case
    env = {"FAR_RING_MIN_ROWS": "1"} if kern == "ring" else {}
    if kern == "direct":
        env["FAR_PREFILL_KERNEL"] = "0"
    fwd = _ctx_with_env(dict(env, FAR_TENSOR_REVERSE="0"))
    rev = _ctx_with_env(dict(env, FAR_TENSOR_REVERSE="1"))
    try:
        if kern != "auto":
            far.far_set_regime(fwd, far.FAR_REGIME_PREFILL)
            far.far_set_regime(rev, far.FAR_REGIME_PREFILL)
        inp = random_inputs(W, T, H, seed=900 + T)
        g = to_gpu(inp)
        for norm in (True, False):
            a = run_gpu(fwd, g, 1e-6, 0.0, 3, guard=256, want_norm=norm)
            b = run_gpu(rev, g, 1e-6, 0.0, 3, guard=256, want_norm=norm)
            for k in a:
                assert np.array_equal(a[k], b[k]), k
            ref = run_oracle(inp, "bf16", 1e-6, 0.0, 3, want_norm=norm)
            log("tensor order %s norm=%d" % (case, norm),
                compare(b, ref, "bf16", exact_saturation=False))
    finally:
        fwd.close()
        rev.close()


def test_per_tensor_fp8_row_range_and_full_size(ctx):
    # rows [100, 3000) of the Gemma workload: the scale covers those rows only
    wl = WORKLOADS["c5_gemma_fp8_token_bf16"]
    inp = make_inputs(wl)
    g = to_gpu(inp)
    for norm in (True, False):
        got = run_gpu(ctx, g, wl.eps, wl.weight_bias, 3, rows=(100, 3000), want_norm=norm)
        ref = run_oracle(inp, "bf16", wl.eps, wl.weight_bias, 3, rows=(100, 3000), want_norm=norm)
        log("tensor c5 rows norm=%d" % norm,
            compare(got, ref, "bf16", rows=slice(100, 3000), exact_saturation=False))
        assert not got["quant_out"][:100].any() and not got["quant_out"][3000:].any()
        assert not got["residual_out"][:100].any() and not got["residual_out"][3000:].any()
    # all rows, in the launch configuration of a full-size call
    got = run_gpu(ctx, g, wl.eps, wl.weight_bias, 3)
    ref = run_oracle(inp, "bf16", wl.eps, wl.weight_bias, 3)
    log("tensor c5 full", compare(got, ref, "bf16", exact_saturation=False))


def test_per_tensor_fp8_errors(ctx):
    inp = random_inputs(2, 16, 256, seed=77)
    g = to_gpu(inp)
    q = torch.empty(16, 256, dtype=torch.uint8, device="cuda")
    sc = torch.empty(1, dtype=torch.float32, device="cuda")
    small = torch.empty(far.far_fp8_tensor_workspace_bytes(16) - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(far.FarError) as e:
        far.far_fused_fp8_tensor(ctx, g["partials"], g["residual"], g["gamma"], 1e-6,
                                 quant_out=q, scale_out=sc, workspace=small)
    assert e.value.status == far.FAR_ERR_INVALID_ARG
    ws = torch.empty(far.far_fp8_tensor_workspace_bytes(16) + 512, dtype=torch.uint8, device="cuda")
    with pytest.raises(far.FarError) as e:
        far.far_fused_fp8_tensor(ctx, g["partials"], g["residual"], g["gamma"], 1e-6,
                                 quant_out=q, scale_out=sc, workspace=ws[16:])
    assert e.value.status == far.FAR_ERR_ALIGNMENT
    # the workspace may not overlap an output
    big = torch.empty(16 * 256 + far.far_fp8_tensor_workspace_bytes(16), dtype=torch.uint8, device="cuda")
    with pytest.raises(far.FarError) as e:
        far.far_fused_fp8_tensor(ctx, g["partials"], g["residual"], g["gamma"], 1e-6,
                                 quant_out=big[:16 * 256].view(16, 256), scale_out=sc,
                                 workspace=big)
    assert e.value.status == far.FAR_ERR_INVALID_ARG
    # far_fused refuses the per-tensor pattern (it has no workspace)
    with pytest.raises(far.FarError) as e:
        far.far_fused(ctx, g["partials"], g["residual"], g["gamma"], 1e-6, 0.0, 3,
                      quant_out=q, scale_out=torch.empty(16, dtype=torch.float32, device="cuda"))
    assert e.value.status == far.FAR_ERR_INVALID_ARG


def test_per_tensor_fp8_repeated_in_a_graph(ctx):
    """The memset and both passes are captured; replaying reuses the
    workspace and gives the same bits."""
    inp = random_inputs(4, 700, 4096, seed=88)
    g = to_gpu(inp)
    T, H = 700, 4096
    q = torch.empty(T, H, dtype=torch.uint8, device="cuda")
    sc = torch.empty(1, dtype=torch.float32, device="cuda")
    rout = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(far.far_fp8_tensor_workspace_bytes(T), dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    kw = dict(quant_out=q, scale_out=sc, workspace=ws, residual_out=rout, stream=s)
    far.far_fused_fp8_tensor(ctx, g["partials"], g["residual"], g["gamma"], 1e-6, **kw)
    torch.cuda.synchronize()
    q0, s0 = q.clone(), sc.clone()
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gr, stream=s):
        far.far_fused_fp8_tensor(ctx, g["partials"], g["residual"], g["gamma"], 1e-6, **kw)
    q.zero_()
    for _ in range(3):
        with torch.cuda.stream(s):
            gr.replay()
    torch.cuda.synchronize()
    far.far_check(ctx)
    assert torch.equal(q, q0) and torch.equal(sc, s0)
    del gr


def test_prepared_call_replays_on_new_contents(ctx):
    """far.FarCall marshals once; each call uses the buffers' current contents."""
    inp = random_inputs(8, 16, 4096, seed=61)
    g = to_gpu(inp)
    T, H = 16, 4096
    rout = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    q = torch.empty(T, H, dtype=torch.uint8, device="cuda")
    sc = torch.empty(T, dtype=torch.float32, device="cuda")
    call = far.FarCall(ctx, g["partials"], g["residual"], g["gamma"], 1e-6, 1.0, 2,
                       residual_out=rout, quant_out=q, scale_out=sc)
    for k in range(3):
        fresh = random_inputs(8, 16, 4096, seed=62 + k)
        for dst, src in zip(g["partials"], fresh["partials"]):
            dst.copy_(src)
        call()
        torch.cuda.synchronize()
        from reduce_residual_add_b200.inputs import as_u16
        got = {"residual_out": as_u16(rout.cpu()), "norm_out": None,
               "quant_out": q.cpu().numpy(), "scale_out": sc.cpu().numpy()}
        ref = run_oracle({"partials": fresh["partials"], "residual": inp["residual"],
                          "gamma": inp["gamma"]}, "bf16", 1e-6, 1.0, 2, want_norm=False)
        compare(got, ref, "bf16")


def test_bounded_wait_gives_up_reports_timeout_and_context_stays_usable(kctx):
    """Make a wait run out: the ring producer skips one bulk copy (a barrier
    that nothing completes).  The consumers' wait gives up after 20 ms, the
    kernel still ends, far_check reports FAR_ERR_TIMEOUT, and the next call
    on the same context is correct."""
    c = kctx["ring"]
    inp = random_inputs(4, 600, 4096, seed=71)
    g = to_gpu(inp)
    assert far.far_describe_launch(c, 600, 4096, torch.bfloat16, 4, True)["kernel"] == 1
    far.far_test_stall(c, 7, 20000)        # segment 7 of each CTA with two rows or more
    try:
        rout = torch.empty(600, 4096, dtype=torch.bfloat16, device="cuda")
        nout = torch.empty_like(rout)
        far.far_fused(c, g["partials"], g["residual"], g["gamma"], 1e-6, 0.0, 0,
                      residual_out=rout, norm_out=nout)
        torch.cuda.synchronize()
        with pytest.raises(far.FarError) as e:
            far.far_check(c)
        assert e.value.status == far.FAR_ERR_TIMEOUT
    finally:
        far.far_test_stall(c, -1, 0)
    far.far_check(c)                       # the word was cleared
    got = run_gpu(c, g, 1e-6, 0.0, 0)
    ref = run_oracle(inp, "bf16", 1e-6, 0.0, 0)
    compare(got, ref, "bf16")


def test_per_tensor_fused_alongside_other_work(kctx, ctx):
    """The one-launch per-tensor form waits for rows, not for CTAs: with
    GEMMs holding SMs on another stream while it runs (so its CTAs start as
    those free up), it completes, no wait gives up, and its outputs match
    the oracle."""
    c = kctx["ring_fused"]
    W, T, H = 4, 2048, 8192
    inp = random_inputs(W, T, H, dtype="bf16", seed=4242, has_residual=True)
    g = to_gpu(inp)
    a = torch.randn(8192, 8192, device="cuda", dtype=torch.bfloat16)
    side = torch.cuda.Stream()
    torch.cuda.synchronize()
    with torch.cuda.stream(side):
        for _ in range(24):
            b = a @ a
    got = run_gpu(c, g, 1e-6, 0.0, 3, guard=512, want_norm=False)
    ref = run_oracle(inp, "bf16", 1e-6, 0.0, 3, want_norm=False)
    st = compare(got, ref, "bf16")
    log("tensor fused alongside GEMMs", st)
    assert st["quant_out"][1] > 0.95
    del b


def test_per_tensor_fused_bounded_waits(kctx):
    """Per-tensor FP8 in one ring launch (both passes, a bounded wait for
    every row between them): a skipped bulk copy makes the consumers' wait
    give up, so not every row is done and the wait between the passes gives
    up too; the kernel ends, far_check reports FAR_ERR_TIMEOUT, and the next
    call on the context is correct."""
    c = kctx["ring_fused"]
    # more rows than the grid has CTAs (at most 8 per SM): the first pass
    # deals rows from a counter, so some CTA takes two rows or more, and
    # its copy 7 (in its second row: 5 segments per row) is skipped
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    T, H = 9 * sms, 4096
    assert far.far_describe_launch(c, T, H, torch.bfloat16, 4, True, pattern=3)["grid_ctas"] < T
    inp = random_inputs(4, T, H, seed=72)
    g = to_gpu(inp)
    q = torch.empty(T, H, dtype=torch.uint8, device="cuda")
    sc = torch.empty(1, dtype=torch.float32, device="cuda")
    rout = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(far.far_fp8_tensor_workspace_bytes(T), dtype=torch.uint8, device="cuda")
    far.far_test_stall(c, 7, 20000)
    try:
        far.far_fused_fp8_tensor(c, g["partials"], g["residual"], g["gamma"], 1e-6, 0.0,
                                 quant_out=q, scale_out=sc, workspace=ws, residual_out=rout)
        torch.cuda.synchronize()
        with pytest.raises(far.FarError) as e:
            far.far_check(c)
        assert e.value.status == far.FAR_ERR_TIMEOUT
    finally:
        far.far_test_stall(c, -1, 0)
    far.far_check(c)
    got = run_gpu(c, g, 1e-6, 0.0, 3, want_norm=False)
    ref = run_oracle(inp, "bf16", 1e-6, 0.0, 3, want_norm=False)
    compare(got, ref, "bf16", exact_saturation=False)


@pytest.mark.parametrize("kern", ["ring", "direct", "decode"])
def test_format_edges_overflow_and_subnormals(kctx, kern):
    """fp16: partials of 30000 sum past 65504; y, held in fp32, stays finite,
    so the new residual rounds to +inf in fp16 while the normalised output is
    finite, on both sides.  bf16 / fp16: gamma in the subnormal range gives
    subnormal normalised outputs, which must be kept, not flushed."""
    c = kctx[kern]
    T, H = 300 if kern != "decode" else 8, 4096
    # overflow rows: fp16 partials of 30000 in the first columns of some rows
    inp = random_inputs(4, T, H, dtype="fp16", seed=91)
    for p in inp["partials"]:
        p[::7, :16] = 30000.0
    got = run_gpu(c, to_gpu(inp), 1e-6, 0.0, 0)
    ref = run_oracle(inp, "fp16", 1e-6, 0.0, 0)
    compare(got, ref, "fp16")
    assert np.all(got["residual_out"][::7, :16] == 0x7C00)          # +inf
    # subnormal outputs: gamma around 2^-130 (bf16) / 2^-20 (fp16)
    for dt, tiny in (("bf16", 2.0 ** -130), ("fp16", 2.0 ** -20)):
        inp = random_inputs(3, T, H, dtype=dt, seed=92)
        tdt = torch.bfloat16 if dt == "bf16" else torch.float16
        inp["gamma"] = (torch.rand(H, generator=torch.Generator().manual_seed(5)) * tiny).to(tdt)
        got = run_gpu(c, to_gpu(inp), 1e-6, 0.0, 0)
        ref = run_oracle(inp, dt, 1e-6, 0.0, 0)
        compare(got, ref, dt)
        exp = (got["norm_out"].astype(np.int64) >> (7 if dt == "bf16" else 10)) & (0xFF if dt == "bf16" else 0x1F)
        assert np.mean(exp == 0) > 0.5                               # mostly subnormal, kept



# ---------------------------------------------------------------------------
# per-group FP8
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("kern", ["ring", "ring_l1", "direct", "auto"])
@pytest.mark.parametrize("case", [
    (2, 8, 64, 8, "bf16"),          # one pack per group; rows inside a warp
    (2, 8, 64, 64, "fp16"),         # one group per row
    (3, 40, 256, 16, "bf16"),
    (4, 300, 8192, 128, "bf16"),
    (8, 150, 7168, 128, "fp16"),
    (2, 30, 16384, 256, "bf16"),    # 2048 packs: one CTA of 512 consumers
    (3, 200, 12288, 128, "bf16"),   # 1536 packs: 384 consumers
    (8, 60, 10240, 64, "fp16"),     # 1280 packs: 320 consumers
    (5, 70, 1000, 8, "bf16"),       # ragged H: 125 packs
    (8, 4, 4096, 32, "bf16"),       # decode-sized
], ids=lambda c: "W%d_T%d_H%d_G%d_%s" % c)
def test_per_group_fp8(kctx, ctx, case, kern):
    W, T, H, G, dt = case
    c = ctx if kern == "auto" else kctx[kern]
    inp = random_inputs(W, T, H, dtype=dt, seed=700 + W + T + H + G)
    got = run_gpu(c, to_gpu(inp), 1e-6, 0.0, 4, group=G, guard=512)
    ref = run_oracle(inp, dt, 1e-6, 0.0, 4, group=G)
    log("group %s %s" % (kern, case), compare(got, ref, dt))


def test_per_group_full_size_sampled(ctx):
    wl = WORKLOADS["c4_prefill_fp8_static"]
    inp = make_inputs(wl)
    got = run_gpu(ctx, to_gpu(inp), wl.eps, 0.0, 4, group=128)
    rows = _sample_rows(wl.T, inp["outlier_rows"].tolist(), 120, 5)
    ref = run_oracle(inp, "bf16", wl.eps, 0.0, 4, row_list=rows, group=128)
    log("group c4 full", compare(got, ref, "bf16", rows=rows))
    q = (got["quant_out"] & 0x7F).reshape(wl.T, wl.H // 128, 128)
    assert np.all(np.any(q == 0x7E, axis=2))


def test_per_group_errors(ctx):
    inp = random_inputs(2, 4, 2048, seed=78)
    g = to_gpu(inp)
    q = torch.empty(4, 2048, dtype=torch.uint8, device="cuda")
    for G in (24, 512, 4):
        sc = torch.empty(4 * 2048 // 4, dtype=torch.float32, device="cuda")
        with pytest.raises(far.FarError) as e:
            lib = far.lib()
            import ctypes
            arr = (ctypes.c_void_p * 2)(*[p.data_ptr() for p in g["partials"]])
            st = lib.far_fused_fp8_group(ctx.handle, 0, 4, arr, 2, ctypes.c_void_p(g["residual"].data_ptr()),
                                         None, ctypes.c_void_p(g["gamma"].data_ptr()), 4, 2048, 0, 1e-6,
                                         0.0, G, None, ctypes.c_void_p(q.data_ptr()),
                                         ctypes.c_void_p(sc.data_ptr()), None)
            if st != far.FAR_OK:
                raise far.FarError(st)
        assert e.value.status == far.FAR_ERR_UNSUPPORTED
    with pytest.raises(far.FarError) as e:
        far.far_fused(ctx, g["partials"], g["residual"], g["gamma"], 1e-6, 0.0, 4, quant_out=q,
                      scale_out=torch.empty(4, dtype=torch.float32, device="cuda"))
    assert e.value.status == far.FAR_ERR_INVALID_ARG
