"""bench.py keeps its JSON contract: one line with the metric, the roofline of
the attention kernel, the CPU baseline, the end-to-end figure, the launch
count and the clocks sampled in the timed region (short run on one GPU)."""
import json
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_bench_json_line():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--steps", "3", "--warmup", "3",
                          "--e2e-steps", "2", "--no-dense", "--cpu-budget", "2"],
                         capture_output=True, text=True, timeout=900, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "cpu_baseline", "e2e",
                "gpu_launches", "clocks"):
        assert key in d, key
    assert d["n_gpus"] == 1 and d["steps"] == 3 and d["warmup"] >= 3 and d["value"] > 0
    assert d["config"]["workload"] and d["config"]["kept_pairs"] > 0
    r = d["roofline"]
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and 0 < r["frac"] < 1.5
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-9
    c = d["cpu_baseline"]
    assert c["kind"] == "oracle" and c["value"] > 0 and c["cores"] >= 1
    e = d["e2e"]
    assert e["value"] > 0 and e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    # pool, tensor-core scores, select, scan, fill, attention: six kernels of
    # this library per step, as CUPTI recorded them
    assert d["gpu_launches"] == 3 * 6
    if d["gpu_launches_source"].startswith("cupti"):
        ks = d["step_kernels"]
        assert len(ks) == 6 and all(k.startswith("sta::") for k in ks), ks
        assert sum("attn_fwd_kernel" in k for k in ks) == 1 and sum("score_tc_kernel" in k for k in ks) == 1
    assert d["clocks"]["sm_mhz"] is not None and isinstance(d["clocks"]["reasons"], list)
    b = d["build_roofline"]
    assert b["bound"] == "hbm" and b["unit"] == "GB/s" and 0 < b["frac"] < 1.5
    assert abs(b["frac"] - b["achieved"] / b["peak"]) < 1e-9
    assert abs(r["frac_burst"] - r["achieved"] / r["peak_burst"]) < 1e-9
    # every other layer of the workload table: 480p, 129 frames at four
    # densities, the reuse layer at five
    rows = d["per_config"]
    assert [x["workload"].split("_")[0] for x in rows] == ["dit480p"] + ["dit720p129f"] * 4 + ["reuse"] * 5, \
        [x["workload"] for x in rows]
    for x in rows:
        assert x["attn_ms"] > 0 and x["build_ms"] > 0 and x["kept_pairs"] > 0
        assert 0 < x["frac_burst"] <= x["frac_sustained"] < 1.5 and 0 < x["pairing_efficiency"] <= 1.0
        assert isinstance(x["clocks"]["reasons"], list)
    # the reuse rows run the overlap pairing, which never does worse than the
    # frame pairing it is compared with
    for x in rows[-5:]:
        assert x["pairing"].startswith("overlap")
        assert x["pairing_efficiency"] >= x["pairing_efficiency_frames"] - 1e-12
