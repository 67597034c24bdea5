"""The reference arm of bench.py (the fp64 oracle on the host cores) prints
one JSON line with the contract's keys; runs on the CPU."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--config", "0", "--steps", "1", "--warmup", "3"],
                         capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 1 and d["warmup"] == 3
    assert d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["config"]["workload"].startswith("tiny-linear-4e-2x2")


def test_warmup_below_three_is_refused():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--place", "--warmup", "2"],
                         capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode != 0 and "at least 3 warm-up steps" in out.stderr


def test_traffic_table_keyed_to_kernel_sources(tmp_path, monkeypatch):
    """roofline.traffic comes from profiles/traffic.json only while the captured
    kernel's listed sources hash to the stored value; a change to another CUDA
    file does not void it, a change to a listed one does."""
    sys.path.insert(0, ROOT)
    import bench
    import synth

    csrc = tmp_path / "tiled_rank_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    (csrc / "k.cu").write_text("kernel v1")
    (csrc / "h.cuh").write_text("header")
    (csrc / "other.cu").write_text("unrelated v1")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    cfg = synth.CONFIGS[1]
    sha = bench.source_sha(["k.cu", "h.cuh"])
    table = {f"gateup:{cfg.name}:T=64": {"dram_bytes_per_launch": 123, "sources": ["k.cu", "h.cuh"], "source_sha": sha}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(table))
    assert bench.traffic_for("gateup", 64, cfg) == 123
    assert bench.traffic_for("gateup", 8, cfg) is None
    (csrc / "other.cu").write_text("unrelated v2")
    assert bench.traffic_for("gateup", 64, cfg) == 123
    (csrc / "k.cu").write_text("kernel v2")
    assert bench.traffic_for("gateup", 64, cfg) is None


def test_clock_sampler_with_a_fake_nvml(monkeypatch):
    """The clocks block of the bench line from NVML reads alone: the median SM
    clock of the samples, the maximum clock, and the event reasons seen (the
    idle bit dropped); without NVML it says so instead of inventing clocks."""
    import types
    import time
    sys.path.insert(0, ROOT)
    import bench

    clocks = iter([1965, 1700, 1800] * 100000)
    fake = types.SimpleNamespace(
        NVML_CLOCK_SM=1,
        nvmlInit=lambda: None,
        nvmlDeviceGetHandleByPciBusId=lambda bus: (_ for _ in ()).throw(RuntimeError("no bus id")),
        nvmlDeviceGetHandleByIndex=lambda i: ("gpu", i),
        nvmlDeviceGetMaxClockInfo=lambda h, kind: 1965,
        nvmlDeviceGetClockInfo=lambda h, kind: next(clocks),
        nvmlDeviceGetCurrentClocksEventReasons=lambda h: 0x1 | 0x4,
    )
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    with bench.ClockSampler(0) as s:
        while len(s.samples) < 30:
            time.sleep(0.001)
    r = s.report()
    assert r["sm_mhz"] == 1800.0 and r["sm_max_mhz"] == 1965.0 and r["samples"] >= 30
    assert r["reasons"] == ["sw_power_cap"]

    fake.nvmlDeviceGetCurrentClocksEventReasons = lambda h: 0x8 | 0x40
    with bench.ClockSampler(0) as s:
        while len(s.samples) < 3:
            time.sleep(0.001)
    assert s.report()["reasons"] == ["hw_slowdown", "hw_thermal_slowdown"]

    monkeypatch.setitem(sys.modules, "pynvml", None)      # import fails: no NVML
    r = bench.ClockSampler(0).report()
    assert r["sm_mhz"] is None and r["reasons"] == ["unavailable"]


def test_reference_arm_under_torchrun_two_ranks():
    """Launched like the driver's N=2 reference arm: rank 0 alone runs the
    oracle and prints one line; the other rank exits 0 without work; the
    oracle's BLAS uses the host cores although torchrun sets OMP_NUM_THREADS=1."""
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    out = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
                          "--master-addr", "127.0.0.1", "--master-port", str(port),
                          os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                          "--config", "0", "--steps", "1", "--warmup", "3"],
                         capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2
    cb = d["cpu_baseline"]
    assert cb["blas_threads"] == cb["cores"] == len(os.sched_getaffinity(0))
