"""Host-side pieces of bench.py that need no GPU."""
from __future__ import annotations

import json
import os
import time

import bench
from reduce_residual_add_b200.inputs import WORKLOADS, make_inputs


def test_algorithmic_bytes_of_the_workloads():
    c4 = WORKLOADS["c4_prefill_fp8_static"]
    assert bench.algorithmic_bytes(c4, c4.T, False) == 872_431_616
    assert bench.algorithmic_bytes(c4, c4.T, True) == 1_006_649_344
    c5 = WORKLOADS["c5_gemma_fp8_token_bf16"]
    assert bench.algorithmic_bytes(c5, c5.T, False) == 616_593_408
    assert bench.algorithmic_bytes(c5, c5.T, True) == 675_313_664
    c4t = WORKLOADS["c4_prefill_fp8_tensor"]
    assert bench.algorithmic_bytes(c4t, c4t.T, False) == 872_431_616 + 4
    c4g = WORKLOADS["c4_prefill_fp8_group128"]
    assert bench.algorithmic_bytes(c4g, c4g.T, False) == 872_431_616 + 4 * 8192 * 64
    c3 = WORKLOADS["c3_3d"]
    assert bench.algorithmic_bytes(c3, c3.T, True) == 20_975_616
    c1 = WORKLOADS["c1_small"]
    assert bench.algorithmic_bytes(c1, c1.T, True) == 5_248
    for T, b in ((1, 98_304), (8, 729_088), (32, 2_891_776), (80, 7_217_152)):
        wl = WORKLOADS["c2_decode_T%d" % T]
        assert bench.algorithmic_bytes(wl, T, True) == b


def test_touched_bytes_and_rotation_size():
    # a rotation cycle must touch more than 2x L2 for the cold timings
    for name in ("c2_decode_T1", "c2_decode_T80", "c3_3d"):
        wl = WORKLOADS[name]
        per = bench.touched_bytes(wl, True)
        n = max(2, -(-2 * bench.L2_BYTES // per))
        assert n * per >= 2 * bench.L2_BYTES
    assert bench.touched_bytes(WORKLOADS["c3_3d"], True) == 20_975_616 - 2048 * 2


def test_clock_sampler_starts_and_stops_without_a_gpu():
    s = bench.ClockSampler(0, period_s=0.001)
    s.start()
    time.sleep(0.01)
    out = s.stop()
    assert set(out) >= {"sm_mhz", "sm_max_mhz", "reasons"}


def test_peak_and_traffic_lookup():
    peak, kind = bench.hbm_peak()
    assert peak > 1000 and kind in ("measured", "fallback")
    # the traffic figure is only used while the kernel source is unchanged
    t = bench.profiled_traffic("c4_prefill_fp8_static")
    path = os.path.join(bench.ROOT, "profiles", "traffic.json")
    if os.path.exists(path):
        d = json.load(open(path))
        e = d.get("c4_prefill_fp8_static")
        if e and e.get("source_sha256") == bench.kernel_source_hash():
            assert t == e["traffic_bytes_per_launch"]
        else:
            assert t is None
    else:
        assert t is None


def test_workload_config_for_every_workload():
    for name, wl in WORKLOADS.items():
        cfg = bench.workload_config(wl, bench.algorithmic_bytes(wl, wl.T, False), False, 1)
        assert "launch" not in cfg
        assert cfg["workload"] == name and cfg["pattern"] in bench.PATTERN_NAMES.values()
        json.dumps(cfg)


def test_cpu_baseline_on_all_cores_and_single_threaded():
    wl = WORKLOADS["c3_3d"].with_(T=96)
    inp = make_inputs(wl)
    out = bench.cpu_baseline(wl, inp, False, budget_s=0.05)
    assert out["kind"] == "oracle" and out["value"] > 0
    assert 1 <= out["cores"] <= bench.host_cores()
    assert out["single_thread"]["cores"] == 1 and out["single_thread"]["value"] > 0
    # per-tensor FP8: one scale over every row, so one thread
    assert bench.oracle_threads(WORKLOADS["c4_prefill_fp8_tensor"], 8192, 64) == 1
    assert bench.oracle_threads(WORKLOADS["c4_prefill_fp8_static"], 5, 64) == 5


def test_reference_arm_line():
    """`bench.py --impl reference` times the oracle on this host and prints
    one JSON line with the CUDA arm's metric, unit and config object."""
    import subprocess
    import sys
    out = subprocess.run([sys.executable, os.path.join(bench.ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "c1_small", "--steps", "3", "--warmup", "3"],
                         capture_output=True, text=True, timeout=300, cwd=bench.ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["unit"] == "GB/s" and line["higher_is_better"] is True and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    wl = WORKLOADS["c1_small"]
    want = bench.workload_config(wl, bench.algorithmic_bytes(wl, wl.T, True), True, 1)
    assert line["config"] == json.loads(json.dumps(want))


def test_kernel_hash_ignores_comments_only():
    a = "int f(int x) { return x + 1; } // one\n/* block */ const char* s = \"// kept\";\n"
    b = "int f(int x) {\n  return x + 1;  // another comment\n}\nconst char* s = \"// kept\";"
    c = "int f(int x) { return x + 2; } const char* s = \"// kept\";"
    d = "int f(int x) { return x + 1; } const char* s = \"// changed\";"
    assert bench.code_tokens(a) == bench.code_tokens(b)
    assert bench.code_tokens(a) != bench.code_tokens(c)
    assert bench.code_tokens(a) != bench.code_tokens(d)
    assert len(bench.kernel_source_hash()) == 64
