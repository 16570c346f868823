"""Host-side pieces of bench.py that decide what its JSON line reports (CPU only):
the ncu traffic figure is used only for the kernel sources it was taken on, the
algorithmic bytes follow the contraction's operand/output/scale sizes, and the
roofline peaks fall back to the recipe's figures when no measured file exists."""
import os
import shutil
import tempfile
import types

import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture
def fake_root(monkeypatch):
    """A throw-away tree (inside the repository's git-ignored _build/) with the
    kernel sources copied, for bench.ROOT to point at."""
    base = os.path.join(ROOT, "_build")
    os.makedirs(base, exist_ok=True)
    d = tempfile.mkdtemp(prefix="bench_root_", dir=base)
    csrc = os.path.join(d, "fp8_block_scaled_bsgemm_b200", "csrc")
    os.makedirs(csrc)
    for f in bench.KERNEL_FILES:
        shutil.copy(os.path.join(ROOT, "fp8_block_scaled_bsgemm_b200", "csrc", f), csrc)
    os.makedirs(os.path.join(d, "profiles"))
    monkeypatch.setattr(bench, "ROOT", d)
    yield d
    shutil.rmtree(d, ignore_errors=True)


def _profile(root, name, sha, workload, traffic):
    with open(os.path.join(root, "profiles", name), "w") as f:
        f.write(f"# summary\n\nkernel_source_sha256: {sha}\nbench_workload: {workload}\n"
                f"traffic_bytes_per_launch: {traffic}\n")


def test_traffic_is_reported_only_for_the_profiled_kernel_sources(fake_root):
    sha = bench.kernel_source_hash()
    assert len(sha) == 16
    _profile(fake_root, "a.md", sha, "square", 34286848)
    _profile(fake_root, "b.md", "0" * 16, "ffn", 99)
    assert bench.profiled_traffic("square") == 34286848
    assert bench.profiled_traffic("ffn") is None            # taken on other sources
    assert bench.profiled_traffic("long_k:128") is None     # never profiled
    # a comment does not change the device code, and keeps the figure
    ptx = os.path.join(fake_root, "fp8_block_scaled_bsgemm_b200", "csrc", "ptx.cuh")
    with open(ptx, "a") as f:
        f.write("\n// edited\n/* a note\n   over two lines */\n")
    assert bench.kernel_source_hash() == sha
    # any change to the code itself unties it
    with open(ptx, "a") as f:
        f.write("\nnamespace bsg { constexpr int kEdited = 1; }\n")
    assert bench.kernel_source_hash() != sha
    assert bench.profiled_traffic("square") is None


def test_malformed_traffic_is_not_reported(fake_root):
    _profile(fake_root, "a.md", bench.kernel_source_hash(), "square", "n/a")
    assert bench.profiled_traffic("square") is None


def test_committed_profiles_name_their_workload_and_sources():
    """Each committed GEMM kernel summary (bsgemm_*.md) carries the three fields
    the bench reads; a quantiser summary (quantize_*.md) the hash of the
    quantiser's code; other summaries (launch lists) the GEMM kernels' hash."""
    paths = [p for p in os.listdir(os.path.join(ROOT, "profiles")) if p.endswith(".md")]
    assert paths
    for p in paths:
        if p.startswith("quantize_"):
            text = open(os.path.join(ROOT, "profiles", p)).read()
            assert "quantiser_source_sha256:" in text and "bench_workload:" not in text, p
            continue
        if not p.startswith("bsgemm_"):
            assert "kernel_source_sha256:" in open(os.path.join(ROOT, "profiles", p)).read(), p
            continue
        text = open(os.path.join(ROOT, "profiles", p)).read()
        for key in ("kernel_source_sha256:", "bench_workload:", "traffic_bytes_per_launch:"):
            assert key in text, (p, key)


def test_algorithmic_bytes_of_the_square_workload():
    p = types.SimpleNamespace(M=4096, N=4096, K=4096, gran=128)
    # A and B codes, BF16 output, FP32 scales [32, 32] per operand
    assert bench.algorithmic_bytes(p) == 2 * 4096 * 4096 + 2 * 4096 * 4096 + 4 * (32 + 32) * 32
    ragged = types.SimpleNamespace(M=1, N=7168, K=7168, gran=128)
    assert bench.algorithmic_bytes(ragged) == 7168 + 7168 * 7168 + 2 * 7168 + 4 * (1 + 56) * 56


def test_peaks_fall_back_without_a_measured_file(monkeypatch):
    base = os.path.join(ROOT, "_build")
    os.makedirs(base, exist_ok=True)
    d = tempfile.mkdtemp(prefix="bench_peaks_", dir=base)
    try:
        monkeypatch.setattr(bench, "ROOT", d)
        pk = bench.measured_peaks()
        assert pk["source"] == "fallback" and pk["hbm_gbs"] == 6650.0 and pk["bf16_tflops"] == 1590.0
        with open(os.path.join(d, "MEASURED_PEAKS.json"), "w") as f:
            f.write('{"hbm_gbs": 7000.5, "bf16_tflops": 1600.25}')
        pk = bench.measured_peaks()
        assert pk == {"hbm_gbs": 7000.5, "bf16_tflops": 1600.25, "source": "measured"}
    finally:
        shutil.rmtree(d, ignore_errors=True)


def test_reference_arm_prints_one_contract_line(capsys, monkeypatch):
    """bench.py --impl reference (the oracle, on host cores) on the tiny
    workload: one JSON line with the contract's keys, no GPU touched."""
    import json
    monkeypatch.delenv("RANK", raising=False)
    bench.main(["--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "0",
                "--cpu-seconds", "0.5"])
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "TFLOP/s"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["config"]["workload"]


def test_reference_arm_runs_on_rank_zero_only(capsys, monkeypatch):
    monkeypatch.setenv("RANK", "1")
    bench.main(["--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "0"])
    assert capsys.readouterr().out.strip() == ""


def test_clock_summary_reports_median_clock_and_active_throttle_reasons():
    """The clocks key: median SM MHz under load, the max clock, and the names of
    the throttle reasons nvidia-smi reported active during the timed region."""
    base = os.path.join(ROOT, "_build")
    os.makedirs(base, exist_ok=True)
    fd, path = tempfile.mkstemp(prefix="clocks_", suffix=".csv", dir=base)
    os.close(fd)
    with open(path, "w") as f:
        f.write("0, 1965, 1965, 700.50, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active\n"
                "0, 1800, 1965, 990.10, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n"
                "0, 1950, 1965, 980.00, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active\n"
                "garbage line\n")
    cs = bench.ClockSampler(0)
    cs.proc, cs.path = object(), path          # as if nvidia-smi had run
    s = cs.summary()
    assert s == {"sm_mhz": 1950.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}
    assert not os.path.exists(path)
    cs2 = bench.ClockSampler(0)                # nvidia-smi missing: no clocks key value
    assert cs2.summary() is None
