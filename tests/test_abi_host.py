"""Host-side checks of the C ABI (no GPU, no compute calls).

The library must load on a machine without a GPU, export every function
include/far.h declares, agree with the header on its constants, and reject
every bad argument on the host (far_validate is the same check far_fused
runs before it launches anything).
"""
from __future__ import annotations

import ctypes
import os
import re
import subprocess

import pytest
import torch

import oracle
from reduce_residual_add_b200 import build as fbuild
from reduce_residual_add_b200 import far

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = open(os.path.join(ROOT, "include", "far.h")).read()


@pytest.fixture(scope="module", autouse=True)
def built():
    fbuild.build()


def declared_functions():
    body = re.sub(r"/\*.*?\*/", "", HEADER, flags=re.S)
    return sorted(set(re.findall(r"\b(far_[a-z0-9_]+)\s*\(", body)))


def test_library_exports_every_declared_function():
    names = declared_functions()
    assert set(names) == set(far.EXPORTS)
    out = subprocess.run(["nm", "-D", "--defined-only", far.lib_path()],
                         capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (far_\w+)", out))
    for n in names:
        assert n in exported, n
        assert hasattr(far.lib(), n)


def _enum(name):
    m = re.search(r"\b%s\s*=\s*(\d+)" % name, HEADER)
    return int(m.group(1))


def test_header_constants_match_binding_and_oracle():
    for n in ("FAR_OK", "FAR_ERR_INVALID_ARG", "FAR_ERR_UNSUPPORTED", "FAR_ERR_ALIGNMENT",
              "FAR_ERR_CUDA", "FAR_ERR_TIMEOUT", "FAR_ERR_INTERNAL", "FAR_BF16", "FAR_FP16",
              "FAR_AR_RESIDUAL_RMSNORM", "FAR_AR_RESIDUAL_RMSNORM_FP8_STATIC",
              "FAR_AR_RESIDUAL_RMSNORM_FP8_TOKEN", "FAR_AR_RESIDUAL_RMSNORM_FP8_TENSOR",
              "FAR_AR_RESIDUAL_RMSNORM_FP8_GROUP",
              "FAR_REGIME_AUTO", "FAR_REGIME_DECODE",
              "FAR_REGIME_PREFILL"):
        assert getattr(far, n) == _enum(n), n
    assert int(re.search(r"#define FAR_MAX_W (\d+)", HEADER).group(1)) == far.FAR_MAX_W
    assert int(re.search(r"#define FAR_MAX_H (\d+)", HEADER).group(1)) == far.FAR_MAX_H
    assert (int(re.search(r"#define FAR_FP8_TENSOR_NOALLOC_MAX_ROWS (\d+)", HEADER).group(1))
            == far.FAR_FP8_TENSOR_NOALLOC_MAX_ROWS)
    # the oracle keeps its own copies of the numbering
    assert (oracle.BF16, oracle.FP16) == (far.FAR_BF16, far.FAR_FP16)
    assert (oracle.AR_RESIDUAL_RMSNORM, oracle.FP8_STATIC, oracle.FP8_TOKEN, oracle.FP8_TENSOR,
            oracle.FP8_GROUP) == (
        far.FAR_AR_RESIDUAL_RMSNORM, far.FAR_AR_RESIDUAL_RMSNORM_FP8_STATIC,
        far.FAR_AR_RESIDUAL_RMSNORM_FP8_TOKEN, far.FAR_AR_RESIDUAL_RMSNORM_FP8_TENSOR,
        far.FAR_AR_RESIDUAL_RMSNORM_FP8_GROUP)
    assert far.far_version() == int(re.search(r"#define FAR_VERSION (\d+)", HEADER).group(1))


def test_status_strings():
    for code in range(7):
        assert far.far_status_string(code).startswith("FAR_")
    assert far.far_status_string(99) == "FAR_ERR_UNKNOWN"


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU path")
def test_create_without_a_gpu_fails_cleanly():
    with pytest.raises(far.FarError) as e:
        far.FarContext(0)
    assert e.value.status == far.FAR_ERR_CUDA


def test_describe_launch_needs_a_context():
    """Both describe calls refuse a NULL context or info before any CUDA call."""
    info = far.far_launch_info()
    L = far.lib()
    assert L.far_describe_launch(None, 8, 4096, far.FAR_BF16, 4, 1, 0, ctypes.byref(info)) == \
        far.FAR_ERR_INVALID_ARG
    for pattern in range(5):
        assert L.far_describe_launch_pattern(None, 8, 4096, far.FAR_BF16, 4, 1, 0, pattern,
                                             ctypes.byref(info)) == far.FAR_ERR_INVALID_ARG


# --------------------------------------------------------------------------
# far_validate on fake, well-spaced addresses (nothing is dereferenced)
# --------------------------------------------------------------------------

T, H, W = 64, 512, 4
TB = T * H * 2
BASE = 1 << 32


def good(**over):
    """A valid argument set: W partials, residual, separate residual_out,
    gamma, norm_out, quant_out, scales, each in its own region."""
    a = dict(row_begin=0, row_end=T, partial_ptrs=[BASE + i * (TB + 4096) for i in range(W)],
             residual=BASE + 100 * TB, residual_out=BASE + 102 * TB, gamma=BASE + 104 * TB,
             T=T, H=H, dtype=far.FAR_BF16, eps=1e-6, weight_bias=0.0,
             pattern=far.FAR_AR_RESIDUAL_RMSNORM_FP8_TOKEN, norm_out=BASE + 106 * TB,
             quant_out=BASE + 108 * TB, scale_in=BASE + 110 * TB, scale_out=BASE + 112 * TB)
    a.update(over)
    return a


def v(**over):
    return far.far_validate(**good(**over))


def test_validate_accepts_good_arguments():
    assert v() == far.FAR_OK
    for p in (0, 1, 2, 3, 4):
        assert v(pattern=p) == far.FAR_OK
    assert v(residual_out=0) == far.FAR_OK                      # in place
    assert v(residual_out=good()["residual"]) == far.FAR_OK     # explicitly in place
    assert v(residual=0) == far.FAR_OK                          # "First" pattern
    assert v(residual=0, residual_out=0) == far.FAR_OK          # norm only
    assert v(pattern=1, norm_out=0) == far.FAR_OK               # norm_out optional with FP8
    assert v(pattern=2, norm_out=0) == far.FAR_OK
    assert v(T=0, row_end=0) == far.FAR_OK                      # empty problem
    assert v(T=0, row_end=0, gamma=0, norm_out=0, quant_out=0, scale_out=0,
             partial_ptrs=[0] * W) == far.FAR_OK                 # ... with NULL buffers
    assert v(row_begin=5, row_end=5) == far.FAR_OK              # empty slice
    assert v(row_begin=16, row_end=48) == far.FAR_OK
    assert v(H=16384, T=1, row_end=1) == far.FAR_OK
    assert v(H=8, T=1, row_end=1) == far.FAR_OK
    assert v(dtype=far.FAR_FP16) == far.FAR_OK
    assert v(eps=0.0) == far.FAR_OK
    assert v(weight_bias=1.0) == far.FAR_OK


@pytest.mark.parametrize("over,status", [
    (dict(W=0), far.FAR_ERR_INVALID_ARG),
    (dict(partial_ptrs=[BASE + i * (TB + 4096) for i in range(17)]), far.FAR_ERR_INVALID_ARG),
    (dict(partial_ptrs=None), far.FAR_ERR_INVALID_ARG),
    (dict(partial_ptrs=[BASE, 0, BASE + 2 * TB + 8192, BASE + 3 * TB + 12288]), far.FAR_ERR_INVALID_ARG),
    (dict(T=-1, row_end=0), far.FAR_ERR_INVALID_ARG),
    (dict(H=0), far.FAR_ERR_INVALID_ARG),
    (dict(H=-8), far.FAR_ERR_INVALID_ARG),
    (dict(H=12), far.FAR_ERR_UNSUPPORTED),
    (dict(H=16392), far.FAR_ERR_UNSUPPORTED),
    (dict(dtype=2), far.FAR_ERR_INVALID_ARG),
    (dict(pattern=5), far.FAR_ERR_INVALID_ARG),
    (dict(pattern=4, quant_out=0), far.FAR_ERR_INVALID_ARG),
    (dict(pattern=4, scale_out=0), far.FAR_ERR_INVALID_ARG),
    (dict(pattern=3, quant_out=0), far.FAR_ERR_INVALID_ARG),
    (dict(pattern=3, scale_out=0), far.FAR_ERR_INVALID_ARG),
    (dict(row_begin=-1), far.FAR_ERR_INVALID_ARG),
    (dict(row_begin=10, row_end=9), far.FAR_ERR_INVALID_ARG),
    (dict(row_end=T + 1), far.FAR_ERR_INVALID_ARG),
    (dict(eps=float("nan")), far.FAR_ERR_INVALID_ARG),
    (dict(eps=float("inf")), far.FAR_ERR_INVALID_ARG),
    (dict(eps=-1e-6), far.FAR_ERR_INVALID_ARG),
    (dict(weight_bias=float("nan")), far.FAR_ERR_INVALID_ARG),
    (dict(gamma=0), far.FAR_ERR_INVALID_ARG),
    (dict(pattern=0, norm_out=0), far.FAR_ERR_INVALID_ARG),
    (dict(pattern=1, quant_out=0), far.FAR_ERR_INVALID_ARG),
    (dict(pattern=1, scale_in=0), far.FAR_ERR_INVALID_ARG),
    (dict(pattern=2, quant_out=0), far.FAR_ERR_INVALID_ARG),
    (dict(pattern=2, scale_out=0), far.FAR_ERR_INVALID_ARG),
    (dict(residual=BASE + 100 * TB + 8), far.FAR_ERR_ALIGNMENT),
    (dict(residual_out=BASE + 102 * TB + 2), far.FAR_ERR_ALIGNMENT),
    (dict(gamma=BASE + 104 * TB + 4), far.FAR_ERR_ALIGNMENT),
    (dict(norm_out=BASE + 106 * TB + 8), far.FAR_ERR_ALIGNMENT),
    (dict(quant_out=BASE + 108 * TB + 8), far.FAR_ERR_ALIGNMENT),
    (dict(scale_out=BASE + 112 * TB + 2), far.FAR_ERR_ALIGNMENT),
    (dict(pattern=1, scale_in=BASE + 110 * TB + 1), far.FAR_ERR_ALIGNMENT),
    (dict(partial_ptrs=[BASE + 8] + [BASE + i * (TB + 4096) for i in range(1, W)]), far.FAR_ERR_ALIGNMENT),
])
def test_validate_rejects(over, status):
    assert v(**over) == status


@pytest.mark.parametrize("name", ["residual_out", "norm_out", "quant_out", "scale_out"])
def test_validate_rejects_outputs_over_inputs(name):
    # each output placed over the first partial, over gamma, and over another output
    g = good()
    assert v(**{name: g["partial_ptrs"][0]}) == far.FAR_ERR_INVALID_ARG
    assert v(**{name: g["gamma"]}) == far.FAR_ERR_INVALID_ARG
    other = "norm_out" if name != "norm_out" else "quant_out"
    assert v(**{name: g[other]}) == far.FAR_ERR_INVALID_ARG


def test_validate_rejects_partial_overlaps():
    g = good()
    # residual written in place over a partial
    assert v(residual=g["partial_ptrs"][1], residual_out=0) == far.FAR_ERR_INVALID_ARG
    # residual_out half-way into the residual (not exactly in place)
    assert v(residual_out=g["residual"] + TB // 2) == far.FAR_ERR_INVALID_ARG
    # quant_out overlapping the tail of norm_out
    assert v(quant_out=g["norm_out"] + TB - 1024) == far.FAR_ERR_INVALID_ARG
    # static scale inside an output
    assert v(pattern=1, scale_in=g["norm_out"] + 64) == far.FAR_ERR_INVALID_ARG
    # ... but a partial read twice is fine (two ranks cannot alias, but reads are harmless)
    assert v(partial_ptrs=[g["partial_ptrs"][0]] * W) == far.FAR_OK


def test_per_tensor_workspace_size():
    assert far.far_fp8_tensor_workspace_bytes(0) == 256
    assert far.far_fp8_tensor_workspace_bytes(1) == 512
    assert far.far_fp8_tensor_workspace_bytes(64) == 512
    assert far.far_fp8_tensor_workspace_bytes(65) == 768
    assert far.far_fp8_tensor_workspace_bytes(8192) == 256 + 4 * 8192


def test_host_staging_bytes():
    """far_host_staging_bytes (host only): gamma + scale header, then two
    buffers of W partials, residual, residual_out, norm_out (2-byte rows),
    FP8 codes and the largest scale block, each part 256-byte aligned."""
    def r256(x):
        return (x + 255) // 256 * 256
    W, H, R = 4, 8192, 100
    seg, codes, scales = r256(R * H * 2), r256(R * H), r256(R * (H // 8) * 4)
    want = r256(H * 2) + 256 + 2 * ((W + 3) * seg + codes + scales)
    assert far.far_host_staging_bytes(W, H, R) == want
    # the default chunk: about 64 MiB of inputs
    dflt = (64 << 20) // ((W + 1) * H * 2)
    assert far.far_host_staging_bytes(W, H, 0) == far.far_host_staging_bytes(W, H, dflt)
    # out of range
    assert far.far_host_staging_bytes(0, H, R) == 0
    assert far.far_host_staging_bytes(17, H, R) == 0
    assert far.far_host_staging_bytes(W, 12, R) == 0
    assert far.far_host_staging_bytes(W, 16392, R) == 0


def test_binding_marshals_host_tensors_for_far_fused_host():
    """The binding's checks for far_fused_host's host tensors (no GPU needed:
    nothing reaches the library before they pass)."""
    import torch
    T, H = 6, 64
    ps = [torch.zeros(T, H, dtype=torch.bfloat16) for _ in range(3)]
    res = torch.zeros(T, H, dtype=torch.bfloat16)
    gam = torch.ones(H, dtype=torch.bfloat16)
    rout = torch.empty(T, H, dtype=torch.bfloat16)
    q = torch.empty(T, H, dtype=torch.uint8)
    sc = torch.empty(T, dtype=torch.float32)
    out = far._args(ps, res, gam, rout, None, q, None, sc, host=True)
    arr, W, _, _, _, T2, H2, dt = out[:8]
    assert (W, T2, H2, dt) == (3, T, H, far.FAR_BF16)
    assert [arr[i] for i in range(3)] == [p.data_ptr() for p in ps]
    # a 3-D view is flattened to (rows, H)
    out3 = far._args([p.view(2, 3, H) for p in ps], res.view(2, 3, H), gam, rout, None, q, None, sc,
                     host=True)
    assert out3[5:7] == (T, H)
    bad = [
        dict(partials=[ps[0], ps[1][:5]]),                               # shapes differ
        dict(partials=[ps[0], ps[1].to(torch.float16)]),                 # dtypes differ
        dict(residual=torch.zeros(T, H, dtype=torch.float16)),          # residual dtype
        dict(residual_out=torch.empty(T, 2 * H, dtype=torch.bfloat16)[:, :H]),   # strided
        dict(quant_out=torch.empty(T, H, dtype=torch.int16)),            # 2-byte codes
        dict(scale_out=torch.empty(T - 1, dtype=torch.float32)),         # too few scales
        dict(gamma=torch.ones(H, dtype=torch.float16)),                  # gamma dtype
        dict(partials=[p.t().contiguous().t() for p in ps]),             # not contiguous
    ]
    base = dict(partials=ps, residual=res, gamma=gam, residual_out=rout, quant_out=q, scale_out=sc)
    for change in bad:
        kw = dict(base, **change)
        with pytest.raises(ValueError):
            far._args(kw["partials"], kw["residual"], kw["gamma"], kw["residual_out"], None,
                      kw["quant_out"], None, kw["scale_out"], host=True)
    # host and device are not mixed: the device marshalling refuses CPU tensors
    with pytest.raises(ValueError):
        far._args(ps, res, gam, rout, None, q, None, sc)
