"""Host-side parts of bench.py that need no GPU: the reference arm's JSON line
(the oracle timed on the host cores) and the parser that turns an ncu CSV of
DRAM byte counters into per-launch traffic figures."""
from __future__ import annotations

import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "2",
                        "--warmup", "1", "--workload", "c1_f32_1024x64"],
                       capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["higher_is_better"] is True
    assert d["steps"] == 2 and d["warmup"] == 1 and d["n_gpus"] == 1 and d["value"] > 0
    assert d["config"]["workload"] == "c1_f32_1024x64" and d["config"]["M"] == 1024
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_is_silent_on_other_ranks():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "1", "--workload", "c1_f32_1024x64"],
                       capture_output=True, text=True, timeout=300, cwd=ROOT, env=env)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_traffic_csv_is_averaged_per_launch(tmp_path, monkeypatch):
    sys.path.insert(0, ROOT)
    import bench

    monkeypatch.setattr(bench, "PROFILES", str(tmp_path))
    hdr = ["ID", "Process ID", "Process Name", "Host Name", "Kernel Name", "Context", "Stream", "Block Size",
           "Grid Size", "Device", "CC", "Section Name", "Metric Name", "Metric Unit", "Metric Value"]
    rows = []
    for launch, (kernel, rd, wr) in enumerate([
            ("void dyt::dyt_bwd_async_kernel<__nv_bfloat16, float, 8, 512, 6, false>(...)", "8.0", "4.0"),
            ("void dyt::dyt_finalize_kernel<float>(...)", "40.0", "2.0"),
            ("void dyt::dyt_bwd_async_kernel<__nv_bfloat16, float, 8, 512, 6, false>(...)", "10.0", "2.0"),
            ("void dyt::dyt_fwd_async_kernel<__nv_bfloat16, float, 8, 512, 8, false>(...)", "1,024.0", "0.0"),
            ("void at::vectorized_elementwise_kernel<...>(...)", "9.0", "9.0")]):
        units = ("Kbyte", "Kbyte") if "finalize" in kernel else ("Mbyte", "Mbyte")
        if "fwd" in kernel:
            units = ("Kbyte", "byte")
        for metric, unit, value in (("dram__bytes_read.sum", units[0], rd), ("dram__bytes_write.sum", units[1], wr)):
            rows.append([str(launch), "1", "python", "h", kernel, "1", "7", "(512, 1, 1)", "(148, 1, 1)", "0", "10.0",
                         "", metric, unit, value])
    csv_path = tmp_path / "traffic.csv"
    with open(csv_path, "w") as f:
        f.write("==PROF== some banner line\n")
        for r in [hdr] + rows:
            f.write(",".join(f'"{c}"' for c in r) + "\n")
    bench.record_traffic(str(csv_path), "case", "ncu ...")
    d = json.load(open(tmp_path / "dram_traffic.json"))["case"]
    assert d["dyt_bwd_kernel"]["launches"] == 2
    assert abs(d["dyt_bwd_kernel"]["bytes_per_launch"] - 12e6) < 1     # (8 + 4 + 10 + 2) MB / 2
    assert abs(d["dyt_finalize_kernel"]["bytes_per_launch"] - 42e3) < 1
    assert abs(d["dyt_fwd_kernel"]["bytes_per_launch"] - 1.024e6) < 1  # thousands separator
    # one backward call: both stage-1 launches (two phases) and its one finalize
    assert abs(d["dyt_backward"]["bytes_per_launch"] - 24.042e6) < 1
    assert d["dyt_backward"]["stage1_launches_per_call"] == 2
    assert all(v["source_hash"] == bench.kernel_source_hash() for v in d.values())
    assert "at::" not in json.dumps(d)


def test_threaded_oracle_baseline_uses_the_host_cores():
    sys.path.insert(0, ROOT)
    import bench
    from synth import workloads

    d = bench.cpu_baseline_threads(workloads.WORKLOADS["c1_f32_1024x64"], seconds_budget=0.5)
    assert d["unit"] == "GB/s" and d["value"] > 0 and d["kind"].startswith("oracle")
    assert 1 <= d["cores"] <= len(os.sched_getaffinity(0))
