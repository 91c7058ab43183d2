"""Benchmark of the exact-attention hot path on B200: one step = one causal prefill of the
MHA workload (B=8, H=32, N=2048, d=128, bf16) through fa_fwd, plus one GQA decode step over
a KV cache (B=32, Hq=32, Hkv=8, lengths uniform in [1024, 8192], d=128) through fa_decode.

Prints ONE JSON line (rank 0).  ``value`` is the prefill throughput in algorithmic TFLOP/s
(4*d flops per unmasked (query, key) pair), summed over ranks; the decode step's KV-cache
GB/s is in ``decode``.  Timing: CUDA events on the launching stream, W untimed warm-up
steps, K timed steps bracketed by a barrier and a synchronize, max over ranks.  Both
workloads' inputs exceed the 126 MB L2, so no flush is needed between steps.

The same line carries a ``configs`` block: every other named workload (the grouped-query
causal prefills at 8K and 32K, the same 8K problem on (batch, sequence, heads, dim) tensors,
sliding window, chunked prefill, paged and FP8 decode, and the small fp32-output problem)
timed the same way, one kernel call per timed iteration, with its roofline fraction; also
the same two prefill problems over FP8 (E4M3) inputs.

``--gpus N``: one process per GPU.  Under torchrun the world size must equal N; started
without torchrun, the script re-launches itself under ``torch.distributed.run`` with N local
ranks.  Every rank runs the same step on its own replica of the workload (no collective on
the data path); times are the max over ranks.

``--impl reference`` times the CPU fp64 oracle (the only reference this method has) on a
bounded row sample of the same prefill workload, on the host cores, with the same metric.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import torch
import torch.distributed as dist

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from exact_io_aware_81_b200 import inputs  # noqa: E402

METRIC = "attn fwd TFLOP/s & % of BF16 peak; decode KV-cache GB/s & % of HBM peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
PREFILL_KERNEL = "fa_prefill_kernel"
DECODE_KERNELS = ("fa_decode_split_kernel", "fa_decode_merge_kernel")


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "exact_io_aware_81_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def load_traffic():
    """DRAM bytes per launch from the committed ncu summary, if it matches these sources."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
    except Exception:
        return {}
    if t.get("source_hash") != kernel_source_hash():
        return {}
    return t.get("kernels", {})


# ------------------------------------------------------------------ clocks sampler

class ClockSampler:
    """Samples SM clock, power and clock-event reasons through NVML in a thread.

    The clock and the reasons are read every ``period_s`` (a few samples fall inside even a
    timed region of well under a second); the power reading, the slowest of the three
    calls, only on every fourth sample (the last reading is repeated in between).
    """

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.period = period_s
        self.samples = []
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            if not uuid.startswith("GPU-"):
                uuid = "GPU-" + uuid
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid.encode())
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # pragma: no cover - depends on the box
            self.err = str(e)

    def _reasons(self, mask):
        nv = self.nv
        names = []
        for attr, name in [("nvmlClocksEventReasonGpuIdle", "gpu_idle"),
                           ("nvmlClocksEventReasonApplicationsClocksSetting", "applications_clocks_setting"),
                           ("nvmlClocksEventReasonSwPowerCap", "sw_power_cap"),
                           ("nvmlClocksEventReasonHwSlowdown", "hw_slowdown"),
                           ("nvmlClocksEventReasonSyncBoost", "sync_boost"),
                           ("nvmlClocksEventReasonSwThermalSlowdown", "sw_thermal_slowdown"),
                           ("nvmlClocksEventReasonHwThermalSlowdown", "hw_thermal_slowdown"),
                           ("nvmlClocksEventReasonHwPowerBrakeSlowdown", "hw_power_brake_slowdown")]:
            bit = getattr(nv, attr, None)
            if bit is None:
                bit = getattr(nv, attr.replace("ClocksEvent", "ClocksThrottle"), None)
            if bit is not None and mask & bit:
                names.append(name)
        return names

    def _run(self):
        nv = self.nv
        pw, n = 0.0, 0
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                try:
                    mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except Exception:
                    mask = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                if n % 4 == 0:
                    pw = nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0
                n += 1
                self.samples.append((time.time(), mhz, pw, self._reasons(mask)))
            except Exception:
                pass
            self._stop.wait(self.period)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()

    def stop(self):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self, t0=None, t1=None):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "note": "NVML unavailable: " + getattr(self, "err", "")}
        s = [x for x in self.samples if (t0 is None or x[0] >= t0) and (t1 is None or x[0] <= t1)]
        if not s:
            s = self.samples[-3:]
        reasons = sorted({r for x in s for r in x[3] if r != "gpu_idle"})
        return {"sm_mhz": statistics.median(x[1] for x in s) if s else None,
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(s),
                "power_w_max": max(x[2] for x in s) if s else None}


# ------------------------------------------------------------------ helpers

def free_port() -> int:
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def relaunch_cmd(n: int, argv, port: int):
    """The torchrun command that starts this script as n local ranks with the same arguments."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
            "--master-addr", "127.0.0.1", f"--master-port={port}", os.path.abspath(__file__), *argv]


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}: start one process per GPU "
                         f"(torchrun --nproc-per-node {args.gpus}), or run without torchrun and let "
                         f"--gpus start the ranks")
    if args.impl == "reference":
        return rank, world, local  # the CPU oracle needs no process group
    if local >= torch.cuda.device_count():
        raise SystemExit(f"bench.py: local rank {local} has no GPU ({torch.cuda.device_count()} visible)")
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return rank, world, local


def max_over_ranks(x: float, world: int, device=None) -> float:
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        dist.barrier()


def oracle_prefill_rate(w, target_s: float, seed: int = 0):
    """Time the oracle on a row sample of prefill workload w sized for about target_s
    seconds; returns (TFLOP/s, seconds, rows_per_head, threads)."""
    import oracle
    B, Hq, Hkv, Nq, Nk, d = w.shape

    def flops_for(rows):
        off = Nk - Nq
        per = sum((min(Nk, r + off + 1) if w.causal else Nk) for r in rows.tolist())
        return 4.0 * d * B * Hq * per

    rows = inputs.sample_rows(Nq, 2, seed=seed, tile=Nq + 1)
    t = time.perf_counter()
    oracle.attn_fwd(w.q, w.k, w.v, w.scale, w.causal, rows=rows)
    dt = max(time.perf_counter() - t, 1e-3)
    rate = flops_for(rows) / dt
    per_row = flops_for(torch.arange(Nq)) / Nq
    n = int(max(1, min(Nq, target_s * rate / per_row)))
    rows = inputs.sample_rows(Nq, n, seed=seed + 1, tile=Nq + 1)
    t = time.perf_counter()
    oracle.attn_fwd(w.q, w.k, w.v, w.scale, w.causal, rows=rows)
    dt = time.perf_counter() - t
    return flops_for(rows) / dt / 1e12, dt, len(rows), oracle.num_threads()


# ------------------------------------------------------------------ reference arm

def step_config(world):
    """The workload of one step, shared by both arms."""
    return {
        "workload": f"{inputs.WORKLOADS[2]} + {inputs.WORKLOADS[5]}",
        "global_batch": 8 * world, "seq_len": 2048, "decode_batch": 32 * world,
        "parallelism": f"replicas: dp{world} (independent problems per GPU, no collective)",
        "l2": "inputs larger than L2 (prefill 537 MB, decode caches 1074 MB)",
    }


def run_reference(args, rank, world):
    out = None
    if rank == 0:
        w = inputs.workload(2)
        # each step: the oracle on a row sample sized for ~args.ref_step_s seconds
        import oracle
        oracle.build()
        rate, dt, nrows, threads = oracle_prefill_rate(w, args.ref_step_s)
        times, flops = [], []
        B, Hq, Hkv, Nq, Nk, d = w.shape
        for i in range(args.warmup + args.steps):
            rows = inputs.sample_rows(Nq, nrows, seed=100 + i, tile=Nq + 1)
            per = sum(min(Nk, r + 1) for r in rows.tolist())
            t = time.perf_counter()
            oracle.attn_fwd(w.q, w.k, w.v, w.scale, True, rows=rows)
            dt = time.perf_counter() - t
            if i >= args.warmup:
                times.append(dt)
                flops.append(4.0 * d * B * Hq * per)
        value = sum(flops) / sum(times) / 1e12
        sample = (f"{nrows} sampled query rows per (b, h) of the prefill workload per step, all 256 (b, h); "
                  "the value is the prefill throughput, as in the other arm (rank 0 only)")
        out = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * sum(times) / len(times), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": step_config(world),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }
        print(json.dumps(out), flush=True)
    return out


# ------------------------------------------------------------------ our arm

def run_ours(args, rank, world, local):
    from exact_io_aware_81_b200 import ops
    ops.load()
    dev = torch.device("cuda", local)
    peaks, peak_src = load_peaks()
    traffic = load_traffic()

    wp = inputs.workload(2)
    wd = inputs.workload(5)
    B, Hq, Hkv, Nq, Nk, d = wp.shape
    q, k, v = wp.q.to(dev), wp.k.to(dev), wp.v.to(dev)
    o = torch.empty((B, Hq, Nq, d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=dev)
    dB, dHq, dHkv, dNmax, dd = wd.shape
    dq, kc, vc, sl = wd.q.to(dev), wd.kcache.to(dev), wd.vcache.to(dev), wd.seqlens.to(dev)
    do = torch.empty((dB, dHq, dd), dtype=torch.bfloat16, device=dev)
    dl = torch.empty((dB, dHq), dtype=torch.float32, device=dev)
    ws = torch.empty(ops.decode_workspace_size(dB, dHq, dNmax, dd), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        ops.fwd(q, k, v, causal=True, scale=wp.scale, out=o, lse=lse, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        ops.decode(dq, kc, vc, sl, scale=wd.scale, workspace=ws, out=do, lse=dl, stream=stream)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    assert ops.get_error() == ops.FA_OK

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.05)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize(dev)
    t0 = time.time()
    for i in range(args.steps):
        step(evs[i])
    torch.cuda.synchronize(dev)
    t1 = time.time()
    barrier(world)
    sampler.stop()
    assert ops.get_error() == ops.FA_OK
    clocks = sampler.summary(t0, t1)

    total_ms = evs[0][0].elapsed_time(evs[-1][2])
    pre_ms = sum(e[0].elapsed_time(e[1]) for e in evs) / args.steps
    dec_ms = sum(e[1].elapsed_time(e[2]) for e in evs) / args.steps
    total_ms = max_over_ranks(total_ms, world, dev)
    pre_ms_max = max_over_ranks(pre_ms, world, dev)
    dec_ms_max = max_over_ranks(dec_ms, world, dev)

    flops = wp.flops()
    dec_bytes = wd.io_bytes()
    pre_tflops = flops / (pre_ms * 1e-3) / 1e12          # this rank, per launch
    dec_gbs = dec_bytes / (dec_ms * 1e-3) / 1e9
    value = world * flops / (pre_ms_max * 1e-3) / 1e12    # whole job
    dec_value = world * dec_bytes / (dec_ms_max * 1e-3) / 1e9

    # ---------------------------------------------------------------- e2e
    e2e = None
    if not args.no_e2e:
        hq, hk, hv = wp.q.pin_memory(), wp.k.pin_memory(), wp.v.pin_memory()
        hdq, hkc, hvc = wd.q.pin_memory(), wd.kcache.pin_memory(), wd.vcache.pin_memory()
        hsl = wd.seqlens.pin_memory()
        ho = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        hl = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
        hdo = torch.empty(do.shape, dtype=do.dtype).pin_memory()
        hdl = torch.empty(dl.shape, dtype=dl.dtype).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hdq, hkc, hvc, hsl))
        d2h = sum(t.numel() * t.element_size() for t in (ho, hl, hdo, hdl))
        e2e_steps = max(1, min(args.steps, args.e2e_steps))

        def e2e_step(ev):
            ev[0].record(stream)
            q.copy_(hq, non_blocking=True); k.copy_(hk, non_blocking=True); v.copy_(hv, non_blocking=True)
            ops.fwd(q, k, v, causal=True, scale=wp.scale, out=o, lse=lse, stream=stream)
            ho.copy_(o, non_blocking=True); hl.copy_(lse, non_blocking=True)
            ev[1].record(stream)
            dq.copy_(hdq, non_blocking=True); kc.copy_(hkc, non_blocking=True)
            vc.copy_(hvc, non_blocking=True); sl.copy_(hsl, non_blocking=True)
            ops.decode(dq, kc, vc, sl, scale=wd.scale, workspace=ws, out=do, lse=dl, stream=stream)
            hdo.copy_(do, non_blocking=True); hdl.copy_(dl, non_blocking=True)
            ev[2].record(stream)

        warm = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        e2e_step(warm)
        torch.cuda.synchronize(dev)
        eev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(e2e_steps)]
        barrier(world)
        torch.cuda.synchronize(dev)
        for i in range(e2e_steps):
            e2e_step(eev[i])
        torch.cuda.synchronize(dev)
        barrier(world)
        e_pre = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in eev) / e2e_steps, world, dev)
        e_dec = max_over_ranks(sum(e[1].elapsed_time(e[2]) for e in eev) / e2e_steps, world, dev)
        # outputs of the e2e run must still match the device-resident run
        assert torch.equal(ho, o.cpu()) and torch.equal(hdo, do.cpu())
        e2e = {"value": world * flops / (e_pre * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
               "ms_per_step": e_pre + e_dec,
               "decode": {"value": world * dec_bytes / (e_dec * 1e-3) / 1e9, "unit": "GB/s"},
               "note": "pinned host buffers; every input of both kernels (q, k, v, q_dec, "
                       "k/v caches, seqlens) is copied H2D and every output D2H each step"}

    # ---------------------------------------------------------------- CPU baseline
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        rate, dt, nrows, threads = oracle_prefill_rate(wp, args.cpu_s)
        cpu = {"value": rate, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": f"{nrows} query rows per (b, h) of the prefill workload (all 256 (b, h)), "
                         f"{dt:.1f} s of fp64 two-pass oracle on {threads} threads"}

    tensor_peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    hbm_peak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    pre_traffic = traffic.get(PREFILL_KERNEL)
    # DRAM bytes per decode step: split kernel (+ merge kernel when it was captured too)
    dec_traffic = None
    if DECODE_KERNELS[0] in traffic:
        dec_traffic = sum(traffic.get(kname, 0) for kname in DECODE_KERNELS)
    result = {
        "metric": METRIC,
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": total_ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": step_config(world),
        "roofline": {
            "bound": "tensor", "achieved": pre_tflops, "peak": tensor_peak, "unit": "TFLOP/s",
            "frac": pre_tflops / tensor_peak, "traffic": pre_traffic,
            "peak_source": f"{peak_src} bf16_tflops (burst, cuBLAS)",
            "kernel": PREFILL_KERNEL, "ms_per_launch": pre_ms,
            "algorithmic_flops_per_launch": flops,
        },
        "decode": {
            "value": dec_value, "unit": "GB/s", "ms_per_step": dec_ms,
            "roofline": {"bound": "hbm", "achieved": dec_gbs, "peak": hbm_peak, "unit": "GB/s",
                         "frac": dec_gbs / hbm_peak, "traffic": dec_traffic,
                         "peak_source": f"{peak_src} hbm_gbs (copy)",
                         "kernel": "+".join(DECODE_KERNELS),
                         "algorithmic_bytes_per_launch": dec_bytes},
        },
        "e2e": e2e,
        "cpu_baseline": cpu,
        "clocks": clocks,
        "gpu_launches": 3 * args.steps,
        "gpu": torch.cuda.get_device_name(dev),
    }
    if not args.no_configs:
        result["configs"] = run_configs(dev, peaks, world)
        result["gpu_launches"] += result["configs"].pop("_launches")
    if rank == 0:
        print(json.dumps(result), flush=True)
    return result


def _time_calls(run, n: int, stream) -> float:
    """Mean milliseconds per call of run() over n calls after 3 warm-up calls, from CUDA
    events recorded on the stream the kernels are launched on."""
    for _ in range(3):
        run()
    e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    torch.cuda.synchronize()
    e[0].record(stream)
    for _ in range(n):
        run()
    e[1].record(stream)
    torch.cuda.synchronize()
    return e[0].elapsed_time(e[1]) / n


def run_configs(dev, peaks, world):
    """Kernel times for every other named workload, one library call per timed iteration:
    prefill 1 (small, fp32 output: launch-bound), the grouped-query causal prefills 3 (also
    on (batch, sequence, heads, dim) tensors through fa_fwd_bshd) and 4, sliding window (6, 8),
    chunked prefill (7, 8), paged decode (9), FP8 decode (10) and FP8 prefill (11, 12).  Every
    input but prefill 1's
    exceeds the 126 MB L2, so back-to-back calls do not hit in L2.  Times are the max over
    ranks; throughputs are per GPU."""
    from exact_io_aware_81_b200 import ops
    tensor_peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    hbm_peak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    stream = torch.cuda.current_stream(dev)
    res, launches = {}, 0
    for kid, bshd in ((1, False), (3, False), (3, True), (4, False), (6, False), (7, False), (8, False)):
        w = inputs.workload(kid)
        B, Hq, Hkv, Nq, Nk, d = w.shape
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=dev)
        if bshd:
            q, k, v = (t.transpose(1, 2).contiguous().to(dev) for t in (w.q, w.k, w.v))
            o = torch.empty((B, Nq, Hq, d), dtype=w.out_dtype, device=dev)
            fwd = ops.fwd_bshd
        else:
            q, k, v = w.q.to(dev), w.k.to(dev), w.v.to(dev)
            o = torch.empty((B, Hq, Nq, d), dtype=w.out_dtype, device=dev)
            fwd = ops.fwd
        n = 50 if kid == 1 else 10
        ms = _time_calls(lambda: fwd(q, k, v, causal=w.causal, scale=w.scale, out_dtype=w.out_dtype, out=o,
                                     lse=lse, window=w.window, stream=stream), n, stream)
        launches += n
        ms = max_over_ranks(ms, world, dev)
        tf = w.flops() / (ms * 1e-3) / 1e12
        entry = {"workload": w.name + ("_bshd" if bshd else ""), "ms": ms, "tflops": tf,
                 "frac": tf / tensor_peak, "bound": "tensor", "algorithmic_flops": w.flops(),
                 "kernel": PREFILL_KERNEL}
        if kid == 1:
            # host cost of one call (binding, C ABI, cached tensor maps, launch), wall clock;
            # the calls only enqueue, and the queue does not fill in 200 calls
            torch.cuda.synchronize()
            t = time.perf_counter()
            for _ in range(200):
                fwd(q, k, v, causal=w.causal, scale=w.scale, out_dtype=w.out_dtype, out=o, lse=lse,
                    window=w.window, stream=stream)
            entry["host_us_per_call"] = (time.perf_counter() - t) / 200 * 1e6
            torch.cuda.synchronize()
            launches += 200
        res[f"workload{kid}" + ("_bshd" if bshd else "")] = entry
        del q, k, v, o, lse, w
        torch.cuda.empty_cache()
    # FP8 prefill (11: workload 2 in E4M3, 12: workload 3 in E4M3).  Its S = Q K^T runs at the
    # FP8 rate and P V at the 16-bit rate, so the bf16 peak is the conservative denominator.
    for kid in (11, 12):
        w = inputs.workload(kid)
        t = [x.to(dev) for x in (w.q, w.k, w.v, w.q_scale, w.k_scale, w.v_scale)]
        B, Hq, Hkv, Nq, Nk, d = w.shape
        o = torch.empty((B, Hq, Nq, d), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=dev)
        n = 10
        ms = _time_calls(lambda: ops.fwd_fp8(*t, causal=w.causal, scale=w.scale, out=o, lse=lse, stream=stream),
                         n, stream)
        launches += n
        ms = max_over_ranks(ms, world, dev)
        tf = w.flops() / (ms * 1e-3) / 1e12
        res[f"workload{kid}"] = {"workload": w.name, "ms": ms, "tflops": tf, "frac": tf / tensor_peak,
                                 "bound": "tensor", "algorithmic_flops": w.flops(), "kernel": PREFILL_KERNEL + " (FP8)",
                                 "peak_note": "bf16 peak: only Q K^T runs at the FP8 rate"}
        del t, o, lse, w
        torch.cuda.empty_cache()
    # decode over a paged cache (9) and over an FP8 cache (10): HBM-bound like decode 5
    for kid in (9, 10):
        w = inputs.workload(kid)
        sl = w.seqlens.to(dev)
        qd = w.q.to(dev)
        B, Hq, d = qd.shape
        out = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=dev)
        ls = torch.empty((B, Hq), dtype=torch.float32, device=dev)
        if kid == 9:
            kp, vp, bt = w.kpages.to(dev), w.vpages.to(dev), w.block_table.to(dev)
            nmax = kp.shape[2] * bt.shape[1]
            wsp = torch.empty(ops.decode_workspace_size(B, Hq, nmax, d), dtype=torch.uint8, device=dev)
            run = lambda: ops.decode_paged(qd, kp, vp, bt, sl, scale=w.scale, workspace=wsp, out=out, lse=ls,
                                           stream=stream)
            kern = "fa_decode_split_kernel (paged) + fa_decode_merge_kernel"
        else:
            kc, vc = w.kcache.to(dev), w.vcache.to(dev)
            ks, vs = w.k_scale.to(dev), w.v_scale.to(dev)
            wsp = torch.empty(ops.decode_workspace_size(B, Hq, kc.shape[2], d), dtype=torch.uint8, device=dev)
            run = lambda: ops.decode_fp8(qd, kc, vc, ks, vs, sl, scale=w.scale, workspace=wsp, out=out, lse=ls,
                                         stream=stream)
            kern = "fa_decode_fp8_kernel + fa_decode_merge_kernel"
        n = 20
        ms = max_over_ranks(_time_calls(run, n, stream), world, dev)
        launches += 2 * n
        gbs = w.io_bytes() / (ms * 1e-3) / 1e9
        res[f"workload{kid}"] = {"workload": w.name, "ms": ms, "gbs": gbs, "frac": gbs / hbm_peak, "bound": "hbm",
                                 "algorithmic_bytes": w.io_bytes(), "kernel": kern}
        del w, run
        torch.cuda.empty_cache()
    assert ops.get_error() == ops.FA_OK
    res["_launches"] = launches
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-s", type=float, default=10.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--ref-step-s", type=float, default=0.5, help="seconds per reference-arm step")
    ap.add_argument("--no-configs", action="store_true", help="skip timing the other named workloads")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        # one process per GPU: start the ranks, and pass on their exit status
        import subprocess
        raise SystemExit(subprocess.call(relaunch_cmd(args.gpus, sys.argv[1:], free_port())))
    rank, world, local = dist_setup(args)
    if args.impl == "reference":
        if rank == 0:  # under torchrun the other ranks exit without work
            run_reference(args, rank, world)
        return
    try:
        run_ours(args, rank, world, local)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
