"""bench.py prints one JSON line with the keys its consumers read: checked for
the reference arm (the CPU oracle, no GPU needed) and for the GPU arm."""

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BASE_KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
             "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"}


def _run(args, timeout):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT, capture_output=True,
                         text=True, timeout=timeout)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1, out.stdout
    return json.loads(lines[0])


def test_reference_arm_line():
    d = _run(["--impl", "reference", "--steps", "2", "--warmup", "3", "--ref-total", "3"], 600)
    assert BASE_KEYS <= set(d)
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["value"] > 0
    assert d["config"]["workload"] == "gpt2_124m"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]


@pytest.mark.gpu
def test_gpu_arm_line():
    d = _run(["--steps", "20", "--warmup", "3", "--grad-sets", "2", "--e2e-steps", "2", "--ref-budget", "1",
              "--ref-budget-1core", "1", "--sweep", "1024,2048", "--cold-steps", "2"], 900)
    assert BASE_KEYS | {"roofline", "gpu_launches", "clocks", "kernels"} <= set(d)
    assert d["n_gpus"] == 1 and d["scaling"] == "weak" and d["higher_is_better"] is True
    r = d["roofline"]
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and 0 < r["frac"] < 1.5
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-9
    assert d["gpu_launches"] == 20 * 2                  # prologue and the chained launch per step
    assert d["e2e"]["h2d_bytes_per_step"] > 0 and d["e2e"]["d2h_bytes_per_step"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle"
    assert set(d["clocks"]) >= {"sm_mhz", "sm_max_mhz", "reasons"}
    assert 0 < r["frac_burst"] < 1.5 and d["cpu_baseline"]["one_core"]["cores"] == 1
    st = d["step_times"]
    assert st["cold_l2_steps"] == 2 and st["ms_cold_l2_median"] > 0 and st["ms_min"] <= st["ms_median"]
    sw = d["sweep"]["n1024"]
    assert sw["matrices"] == 64 and sw["steps"] >= 5 and sw["warmup"] >= 3 and 0 < sw["gemm_frac_burst"] < 1.5
    f8 = d["sweep"]["n2048"]["fp8_variant"]              # e4m3 products run in the per-phase launches
    assert f8["fp8_iters"] == 2 and f8["ms_per_step"] > 0 and f8["ms_per_step_bf16"] > 0
    assert abs(f8["speedup"] - f8["ms_per_step_bf16"] / f8["ms_per_step"]) < 1e-9
    assert "fp8_variant" not in sw                       # the chained launch keeps bf16 operands
    de = d["dense_equivalent"]
    assert de["unit"] == "TFLOP/s" and abs(de["value"] / d["value"] - 1.6307 / 1.1422) < 1e-3


def test_kernel_hash_ignores_comments_but_not_code(tmp_path, monkeypatch):
    import shutil
    sys.path.insert(0, ROOT)
    import bench
    csrc = tmp_path / "muon_newton_schulz_02_b200" / "csrc"
    csrc.mkdir(parents=True)
    for f in ("kernels.cuh", "ptx.cuh"):
        shutil.copy(os.path.join(ROOT, "muon_newton_schulz_02_b200", "csrc", f), csrc / f)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_source_hash()
    k = csrc / "kernels.cuh"
    k.write_text(k.read_text() + "\n// a new comment\n/* and a block\n comment */\n")
    assert bench.kernel_source_hash() == h0
    # the fused small-matrix kernels are not part of the GEMM kernel's record
    text = k.read_text()
    k.write_text(text.replace(bench._FUSED_BEGIN, bench._FUSED_BEGIN + "\nconstexpr int kFusedOnly = 1;\n"))
    assert bench.kernel_source_hash() == h0
    # nor is the prologue
    text = k.read_text()
    k.write_text(text.replace(bench._PRO_BEGIN, bench._PRO_BEGIN + "\nconstexpr int kPrologueOnly = 1;\n"))
    assert bench.kernel_source_hash() == h0
    k.write_text(k.read_text() + "\nconstexpr int kUnused = 1;\n")
    assert bench.kernel_source_hash() != h0


def test_flop_counts_use_the_symmetric_products_once():
    sys.path.insert(0, ROOT)
    import bench
    from muon_newton_schulz_02_b200 import workloads
    k, l = 768, 3072
    per_iter = k * (k + 1) * l + k * k * (k + 1) + 2 * k * k * l      # Gram, polynomial, update
    assert bench.ns_flops([(k, l)]) == 5 * per_iter == bench.ns_flops([(l, k)])
    assert bench.ns_flops([(k, l)], ns_steps=2) == 2 * per_iter
    shapes = workloads.get("gpt2_124m").shapes
    assert sum(bench.flops_by_kind(shapes).values()) == bench.ns_flops(shapes)
    assert abs(bench.ns_flops(shapes) / 1.142e12 - 1) < 5e-3              # the step total the docs quote
    # dense-equivalent: X X^T and A A in full, 2k^2 l + 2k^3 + 2k^2 l per iteration
    assert bench.ns_flops_dense([(k, l)]) == 5 * (4 * k * k * l + 2 * k ** 3) == bench.ns_flops_dense([(l, k)])
    assert abs(bench.ns_flops_dense(shapes) / 1.631e12 - 1) < 5e-3


def test_traffic_is_reported_only_for_the_profiled_kernel_source(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    stored = json.load(open(os.path.join(ROOT, "profiles", "ns_gemm_traffic.json")))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: stored["kernel_source_hash"])
    assert bench.ncu_traffic() == stored["dram_bytes_per_launch_full_workload"]
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0" * 16)
    assert bench.ncu_traffic() is None


def test_peaks_fall_back_when_no_measurement_exists(tmp_path, monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peaks, src = bench.load_peaks()
    assert src == "fallback" and peaks == bench.FALLBACK_PEAKS
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 1.0, "bf16_tflops": 2.0}))
    peaks, src = bench.load_peaks()
    assert src == "measured" and peaks["bf16_tflops"] == 2.0


def test_reference_arm_under_torchrun_prints_once_from_rank_0():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "2", "--warmup", "3", "--ref-total", "2"]
    out = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2
    assert d["cpu_baseline"]["cores"] > 1 or (os.cpu_count() or 1) == 1   # not the launcher's one thread


def test_peak_choice_follows_the_clock_record():
    sys.path.insert(0, ROOT)
    import bench
    peaks = {"bf16_tflops": 1647.8, "bf16_tflops_sustained": 1344.1}
    full = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0}
    capped = {"sm_mhz": 1450.0, "sm_max_mhz": 1965.0}
    assert bench.pick_peak(peaks, full, 5.0)[0] == 1647.8          # full clock: burst
    assert bench.pick_peak(peaks, capped, 0.03)[0] == 1647.8       # short region: burst
    assert bench.pick_peak(peaks, capped, 5.0)[0] == 1344.1        # long region under the cap: sustained
    assert bench.pick_peak({"bf16_tflops": 1590.0}, capped, 5.0)[0] == 1590.0   # no sustained figure
    assert "bf16_tflops_sustained" not in bench.FALLBACK_PEAKS
