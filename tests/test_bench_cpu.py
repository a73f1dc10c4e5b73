"""Host-side checks of the benchmark's bookkeeping (no GPU).

  * the algorithmic work it divides by, against totals written out by hand
    for the 8B-shaped set (parameter counts, nominal Newton-Schulz FLOPs,
    bytes per parameter of each HBM-bound kernel);
  * the one-layer slice is exactly 1/32 of the 32-layer set, which the
    scaled DRAM-traffic figure relies on;
  * the source fingerprint that guards the captured DRAM traffic ignores
    comments and changes with code.
"""
import argparse
import os
import shutil

import bench
from muon_polar_orthogonalized_b200 import workloads as wl

# 8B shapes, written out: per layer Wq, Wo 4096x4096; Wk, Wv 1024x4096;
# gate, up 14336x4096; down 4096x14336; 32 layers; AdamW on two 128256x4096
# tables; bf16 gradients everywhere.
PER_LAYER = [(4096, 4096)] * 2 + [(1024, 4096)] * 2 + [(14336, 4096)] * 2 + [(4096, 14336)]


def test_algorithmic_work_of_the_8b_set():
    w = wl.get("llama_8b_32l")
    work = bench.algorithmic_work(w)
    params = 32 * sum(r * c for r, c in PER_LAYER)
    assert params == 6_979_321_856 == w.muon_params()
    flops = 0
    for r, c in PER_LAYER:
        m, n = min(r, c), max(r, c)
        flops += 32 * (4 * m * m * n + 2 * m ** 3)   # one quintic iteration, nominal
    nominal = 5 * flops
    assert abs(nominal - 665.9e12) < 0.05e12
    got = 5 * (work["gram_flops"] + work["poly_flops"] + work["axpy_flops"])
    assert got == nominal == w.ns_flops_nominal()
    # momentum: bf16 G in (2), fp32 m in and out (8), bf16 X0 out (2)
    assert work["momentum_bytes"] == 12 * params
    # unfused update: bf16 U in (2), fp32 W in and out (8)
    assert work["update_bytes"] == 10 * params
    # AdamW: bf16 g in (2); fp32 p, m, v in and out (24)
    adam_params = 2 * 128256 * 4096
    assert work["adamw_bytes"] == 26 * adam_params


def test_one_layer_slice_is_a_thirty_second_of_the_set():
    full, one = wl.get("llama_8b_32l"), wl.get("llama_8b_1layer")
    a, b = bench.algorithmic_work(full), bench.algorithmic_work(one)
    for k in ("gram_flops", "poly_flops", "axpy_flops", "momentum_bytes", "update_bytes"):
        assert a[k] == 32 * b[k], k
    cap = bench.TRAFFIC_CAPTURES["ns_axpy"]["bytes_per_pass"]
    assert cap["llama_8b_32l"] == 32 * cap["llama_8b_1layer"]


def test_source_fingerprint_ignores_comments_only(tmp_path, monkeypatch):
    src = os.path.join(bench.ROOT, "muon_polar_orthogonalized_b200", "csrc")
    dst = tmp_path / "muon_polar_orthogonalized_b200" / "csrc"
    shutil.copytree(src, dst)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    files = bench.TRAFFIC_CAPTURES["ns_axpy"]["sources"]
    base = bench.source_fingerprint(files)
    current = base == bench.TRAFFIC_CAPTURES["ns_axpy"]["sha"]
    assert (bench.captured_traffic("ns_axpy", "llama_8b_32l") is not None) == current
    f = dst / files[0]
    text = f.read_text()
    f.write_text("// a comment line\n/* and a\n   block comment */\n" + text)
    assert bench.source_fingerprint(files) == base
    assert (bench.captured_traffic("ns_axpy", "llama_8b_32l") is not None) == current
    f.write_text(text.replace("namespace muon {", "namespace muon {\nconstexpr int kProbe = 1;", 1))
    assert bench.source_fingerprint(files) != base
    assert bench.captured_traffic("ns_axpy", "llama_8b_32l") is None


def test_clock_sampler_reads_clocks_and_throttle_reasons(monkeypatch):
    """Median SM clock over the samples that parse, the highest max clock,
    and every throttle reason seen active (nvidia-smi faked)."""
    lines = ["0, 1241, 1965, 985.2, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
             "0, 1300, 1965, 990.1, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
             "0, [N/A], 1965, 990.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
             "0, 1100, 1965, 700.0, 0x0000000000000040, Not Active, Active, Not Active, Not Active",
             "truncated line"]

    class FakeSmi:
        def __init__(self, args, stdout=None, stderr=None):
            assert "--query-gpu=" + bench.ClockSampler.FIELDS in args
            stdout.write("\n".join(lines) + "\n")
            stdout.flush()

        def terminate(self):
            pass

        def wait(self, timeout=None):
            return 0

        def kill(self):
            pass

    monkeypatch.setattr(bench.subprocess, "Popen", FakeSmi)
    sampler = bench.ClockSampler(0)
    sampler.start()
    got = sampler.stop()
    assert got["sm_mhz"] == 1241.0 and got["sm_max_mhz"] == 1965.0 and got["samples"] == 3
    assert got["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]


def test_clock_sampler_without_nvidia_smi(monkeypatch):
    def no_smi(*a, **k):
        raise FileNotFoundError("nvidia-smi")

    monkeypatch.setattr(bench.subprocess, "Popen", no_smi)
    sampler = bench.ClockSampler(0)
    sampler.start()
    got = sampler.stop()
    assert got["sm_mhz"] is None and got["reasons"] == ["nvidia-smi unavailable"]


def test_reference_arm_line_on_small_workload(capsys, monkeypatch):
    """The oracle arm prints one JSON line whose value is the median of its
    per-step samples, with their spread, on the arm's own workload."""
    import json
    import statistics
    monkeypatch.delenv("RANK", raising=False)
    args = argparse.Namespace(workload="single_256x1024", steps=3, warmup=1)
    bench.run_reference(args)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["config"]["workload"] == "single_256x1024"
    cb = line["cpu_baseline"]
    assert len(cb["samples_ms"]) == 3
    assert line["value"] == cb["value"] == round(statistics.median(cb["samples_ms"]), 1)
    assert cb["spread_ms"][0] <= line["value"] <= cb["spread_ms"][1]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["higher_is_better"] is False


def test_cpu_baseline_median_and_spread():
    cb = bench.cpu_baseline(wl.get("single_256x1024"), samples=3)
    assert cb["kind"] == "oracle" and cb["cores"] >= 1
    assert cb["spread_ms"][0] <= cb["value"] <= cb["spread_ms"][1]
    assert cb["extrapolated"] is False   # one matrix and one AdamW tensor: the sample is the step


def test_profile_summary_quotes_the_captured_traffic():
    """The committed ncu summary the bench's DRAM-traffic figure comes from
    names the same source fingerprint and per-layer bytes (the sum of its
    B'X launches' DRAM reads and writes) as bench.TRAFFIC_CAPTURES."""
    import re
    cap = bench.TRAFFIC_CAPTURES["ns_axpy"]
    text = open(os.path.join(bench.ROOT, "profiles", "tc_gemm_pair_llama_8b_1layer.md")).read()
    assert f"`{cap['sha']}`" in text.split("Command")[0]
    per_layer = cap["bytes_per_pass"]["llama_8b_1layer"]
    assert f"{per_layer:,}" in text
    rows = [ln for ln in text.splitlines() if ln.startswith("| ns_axpy")]
    assert len(rows) == 2
    moved = 0
    for ln in rows:
        cells = [c.strip() for c in ln.strip("|").split("|")]
        for c in cells[4:6]:
            m = re.match(r"([0-9][0-9,]*)", c)
            moved += int(m.group(1).replace(",", ""))
    assert moved == per_layer
