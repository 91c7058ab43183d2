"""Host-side logic of bench.py, on the CPU: the clock-record summary (with a stand-in for
NVML), the gate that drops committed DRAM-traffic figures once the kernel sources change,
the max-over-ranks reduction on gloo ranks, and the reference arm (the oracle) end to end."""
import json
import os
import socket
import subprocess
import sys
import tempfile
import types

import pytest
import torch.multiprocessing as mp

import bench

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


def _sampler(samples, max_mhz=1965):
    nv = types.SimpleNamespace(nvmlClocksEventReasonGpuIdle=1, nvmlClocksEventReasonSwPowerCap=4,
                               nvmlClocksEventReasonHwSlowdown=8, nvmlClocksEventReasonSwThermalSlowdown=32)
    s = bench.ClockSampler.__new__(bench.ClockSampler)
    s.ok, s.nv, s.max_mhz = True, nv, max_mhz
    s.samples = [(t, mhz, pw, s._reasons(mask)) for t, mhz, pw, mask in samples]
    return s


def test_clock_reasons_decoded():
    s = _sampler([])
    assert s._reasons(0) == []
    assert s._reasons(1 | 4) == ["gpu_idle", "sw_power_cap"]
    assert s._reasons(8 | 32) == ["hw_slowdown", "sw_thermal_slowdown"]


def test_clock_summary_window_median_and_reasons():
    s = _sampler([(0.0, 1000, 100.0, 1),        # before the timed region: ignored
                  (1.0, 1965, 300.0, 0),
                  (1.1, 1900, 350.0, 4),
                  (1.2, 1965, 320.0, 1),        # gpu_idle is not a throttle reason
                  (9.0, 500, 90.0, 8)])         # after it: ignored
    r = s.summary(0.5, 2.0)
    assert r["sm_mhz"] == 1965 and r["sm_max_mhz"] == 1965 and r["samples"] == 3
    assert r["reasons"] == ["sw_power_cap"] and r["power_w_max"] == 350.0
    # a region shorter than the sampling period falls back to the last samples
    assert _sampler([(0.0, 1800, 1.0, 0), (0.1, 1810, 1.0, 0)]).summary(5.0, 5.001)["samples"] == 2


def test_clock_summary_without_nvml():
    s = bench.ClockSampler.__new__(bench.ClockSampler)
    s.ok, s.err = False, "no NVML"
    r = s.summary()
    assert r["sm_mhz"] is None and r["reasons"] == [] and "no NVML" in r["note"]


def test_traffic_dropped_when_sources_change(monkeypatch):
    with open(os.path.join(ROOT, "profiles", "dram_traffic.json")) as f:
        committed = json.load(f)
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: committed["source_hash"])
    assert bench.load_traffic() == committed["kernels"]
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0" * 16)
    assert bench.load_traffic() == {}


def test_kernel_source_hash_is_stable():
    a, b = bench.kernel_source_hash(), bench.kernel_source_hash()
    assert a == b and len(a) == 16


def test_step_config_weak_scaling():
    c1, c4 = bench.step_config(1), bench.step_config(4)
    assert c1["workload"] == c4["workload"]
    assert c4["global_batch"] == 4 * c1["global_batch"] and c4["decode_batch"] == 4 * c1["decode_batch"]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_max_over_ranks_gloo():
    if HERE not in sys.path:
        sys.path.insert(0, HERE)
    import bench_worker
    with tempfile.TemporaryDirectory() as td:
        path = os.path.join(td, "res.txt")
        mp.start_processes(bench_worker.run, args=(2, _free_port(), path), nprocs=2,
                           start_method="spawn", join=True)
        assert float(open(path).read()) == 2.5


@pytest.mark.slow
def test_reference_arm_runs_on_cpu():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "3",
                        "--ref-step-s", "0.05"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    out = json.loads(r.stdout.strip().splitlines()[-1])
    assert out["impl"] == "reference" and out["value"] > 0 and out["unit"] == "TFLOP/s"
    assert out["config"] == bench.step_config(1) and out["steps"] == 1 and out["warmup"] == 3
    assert out["cpu_baseline"]["kind"] == "oracle" and out["cpu_baseline"]["value"] == out["value"]
    assert out["e2e"]["h2d_bytes_per_step"] == 0 and out["e2e"]["value"] == out["value"]


def _env_without_ranks():
    env = dict(os.environ)
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT", "LOCAL_WORLD_SIZE"):
        env.pop(k, None)
    return env


@pytest.mark.slow
def test_gpus_option_starts_one_rank_per_gpu():
    """`bench.py --gpus 2` started without torchrun re-launches itself as two ranks; the
    reference arm (CPU only) lets this run here: rank 0 prints the one line, with n_gpus 2."""
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--gpus", "2", "--steps", "1",
                        "--warmup", "3", "--ref-step-s", "0.05"], cwd=ROOT, capture_output=True, text=True,
                       timeout=600, env=_env_without_ranks())
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    out = json.loads(lines[0])
    assert out["impl"] == "reference" and out["n_gpus"] == 2
    assert out["config"] == bench.step_config(2)


def test_relaunch_command_is_torchrun_on_loopback():
    cmd = bench.relaunch_cmd(4, ["--gpus", "4", "--steps", "5"], 12345)
    assert cmd[:3] == [sys.executable, "-m", "torch.distributed.run"]
    assert "--nproc-per-node=4" in cmd and "--master-port=12345" in cmd
    assert cmd[cmd.index("--master-addr") + 1] == "127.0.0.1"
    assert cmd[-4:] == ["--gpus", "4", "--steps", "5"] and cmd[-5].endswith("bench.py")


def test_world_size_must_match_gpus():
    env = _env_without_ranks()
    env.update(WORLD_SIZE="2", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--gpus", "1", "--steps", "1",
                        "--warmup", "3"], cwd=ROOT, capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode != 0
    assert "--gpus 1 but WORLD_SIZE=2" in r.stderr
