"""Throughput of the column->row tensor-parallel FFN block on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--mode fused|partials]

One step = one forward of the FFN block (column-parallel GEMM + bias + exact
GeLU, row-parallel GEMM, on-device reduction of the t logical shards + bias +
residual) at M=2048 tokens (batch 4 x seq 512), h=4096, f=16384, t=4, bf16 with
fp32 accumulation, synthetic seeded inputs.  Metric: TFLOP/s with the
algorithmic count 4*M*h*f per step.  Under torchrun each rank runs an
independent replica on its own GPU (its own token batch, no data-path
collective); the value is the total work over all ranks divided by the slowest
rank's device time.

``--impl reference`` times the fp64 CPU oracle instead (on rank 0 only), on a
bounded sample of token rows per step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "TFLOP/s & % of BF16 peak, column→row TP FFN block (t=4 shards), 1 B200"
PROFILES = os.path.join(ROOT, "profiles")


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            p = json.load(fh)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]), "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def _csrc_sha():
    d = os.path.join(ROOT, "megatron_tensor_transformer_bias_b200", "csrc")
    h = hashlib.sha256()
    for f in sorted(os.listdir(d)):
        with open(os.path.join(d, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def _traffic(kernel, units_ratio=1.0):
    """DRAM bytes per launch from the committed ncu capture, or None if the kernel changed since."""
    try:
        with open(os.path.join(PROFILES, "ncu_traffic.json")) as fh:
            t = json.load(fh)
    except Exception:
        return None
    rec = t.get(kernel)
    if not rec or rec.get("csrc_sha") != _csrc_sha():
        return None
    return rec["dram_bytes_per_launch"] * units_ratio


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML (read-only) in a thread."""

    def __init__(self, gpu_index, period_s=0.02):
        self.idx, self.period = gpu_index, period_s
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._t = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(self.idx)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None
            return self
        names = {
            "hw_slowdown": getattr(self.nv, "nvmlClocksEventReasonHwSlowdown", 0x8),
            "hw_thermal_slowdown": getattr(self.nv, "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
            "sw_thermal_slowdown": getattr(self.nv, "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
            "sw_power_cap": getattr(self.nv, "nvmlClocksEventReasonSwPowerCap", 0x4),
            "hw_power_brake": getattr(self.nv, "nvmlClocksEventReasonHwPowerBrakeSlowdown", 0x80),
        }

        def run():
            while not self._stop.is_set():
                try:
                    self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                    r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                    for n, bit in names.items():
                        if r & bit:
                            self.reasons.add(n)
                except Exception:
                    pass
                time.sleep(self.period)

        self._t = threading.Thread(target=run, daemon=True)
        self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._t:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------- CPU oracle timing
def _oracle_rows_flops(n_rows, w):
    return 4 * n_rows * w.h * w.f


def _oracle_setup(w, device):
    import numpy as np
    from megatron_tensor_transformer_bias_b200 import inputs
    p = inputs.ffn_inputs(w.M, w.h, w.f, "bf16", seed=0, device=device)
    c = {k: v.to("cpu", dtype=__import__("torch").float64).numpy() for k, v in p.items()}
    return c


def _oracle_step(c, rows):
    import oracle
    X = c["X"][rows]
    return oracle.ffn_forward(X, c["W1"], c["b1"], c["W2"], c["b2"], X)


def _threads():
    try:
        from threadpoolctl import threadpool_info
        return max(i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas")
    except Exception:
        return os.cpu_count()


def cpu_baseline(w, c, target_s=12.0):
    """The oracle as it stands, on a bounded sample of token rows, timed on the host cores."""
    import numpy as np
    rng = np.random.default_rng(0)
    n0 = 32
    rows = np.sort(rng.choice(w.M, n0, replace=False))
    t0 = time.perf_counter()
    _oracle_step(c, rows)
    t1 = time.perf_counter() - t0
    n = int(min(w.M, max(n0, n0 * target_s / max(t1, 1e-3))))
    rows = np.sort(rng.choice(w.M, n, replace=False))
    t0 = time.perf_counter()
    _oracle_step(c, rows)
    dt = time.perf_counter() - t0
    return {"value": _oracle_rows_flops(n, w) / dt / 1e12, "unit": "TFLOP/s", "cores": _threads(),
            "kind": "oracle",
            "sample": f"{n} of {w.M} token rows of {w.name}, fp64 numpy/OpenBLAS, {dt:.1f} s wall"}


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import numpy as np
    c = _oracle_setup(w, "cpu")
    rng = np.random.default_rng(1)
    rows_per_step = 8
    for _ in range(args.warmup):
        _oracle_step(c, np.sort(rng.choice(w.M, rows_per_step, replace=False)))
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _oracle_step(c, np.sort(rng.choice(w.M, rows_per_step, replace=False)))
    dt = time.perf_counter() - t0
    value = _oracle_rows_flops(rows_per_step, w) * args.steps / dt / 1e12
    sample = f"{rows_per_step} of {w.M} token rows of {w.name} per step, fp64 numpy/OpenBLAS"
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "M": w.M, "h": w.h, "f": w.f, "t": w.t},
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": _threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- GPU arm
def run_ours(args, w):
    import torch
    import torch.distributed as dist

    from megatron_tensor_transformer_bias_b200 import inputs
    from megatron_tensor_transformer_bias_b200 import tpblock as tb

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    tb.lib()
    p = inputs.ffn_inputs(w.M, w.h, w.f, "bf16", seed=0, device=dev)
    if rank:  # each replica runs its own token batch (same weights)
        g = torch.Generator(device=dev).manual_seed(7919 * rank)
        p["X"] = torch.randn(w.M, w.h, generator=g, device=dev).to(torch.bfloat16)
    t = w.t
    W1 = tb.shard_columns(p["W1"], t)
    W2 = tb.shard_rows(p["W2"], t)
    b1 = tb.shard_vector(p["b1"], t)
    X, b2 = p["X"], p["b2"]
    out = torch.empty_like(X)
    mode = tb.MODES[args.mode]
    ws = tb.workspace(tb.tp_ffn_workspace_bytes(w.M, w.h, w.f, t, tb.TP_BF16, mode), dev)
    stream = torch.cuda.current_stream()

    def step():
        tb.tp_ffn_forward(X, W1, b1, W2, b2, X, out, mode=args.mode, ws=ws, stream=stream)

    flops = w.flops
    for _ in range(args.warmup):
        step()
    if tb.tp_get_device_status(stream) != tb.TP_OK:
        raise RuntimeError("device status after warm-up: " + tb.last_error())

    def timed(fn, k):
        barrier()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(k):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        ms = e0.elapsed_time(e1)
        if world > 1:
            tmax = torch.tensor([ms], device=dev, dtype=torch.float64)
            dist.all_reduce(tmax, op=dist.ReduceOp.MAX)
            ms = float(tmax.item())
        return ms

    with ClockSampler(local) as clk:
        # device-resident throughput
        ms = timed(step, args.steps)
        # per-kernel durations over a second timed region, traced with events on the launch stream
        tb.tp_trace_enable(8 * args.steps + 16)
        ms_traced = timed(step, args.steps)
        recs = tb.tp_trace_records()
        tb.tp_trace_disable()
        # end to end through the public API: pinned host X in, host out back, every step
        Xh = X.cpu().pin_memory()
        outh = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        Xd = torch.empty_like(X)
        outd = torch.empty_like(out)

        def step_e2e():
            Xd.copy_(Xh, non_blocking=True)
            tb.tp_ffn_forward(Xd, W1, b1, W2, b2, Xd, outd, mode=args.mode, ws=ws, stream=stream)
            outh.copy_(outd, non_blocking=True)

        for _ in range(3):
            step_e2e()
        ms_e2e = timed(step_e2e, args.steps)
    if tb.tp_get_device_status(stream) != tb.TP_OK:
        raise RuntimeError("device status after timing: " + tb.last_error())

    # per-kernel aggregation of the traced region
    per = {}
    for name, kms in recs:
        d = per.setdefault(name, [0, 0.0])
        d[0] += 1
        d[1] += kms
    dominant = max(per, key=lambda k: per[k][1])
    launches = sum(v[0] for v in per.values())
    dom_avg_ms = per[dominant][1] / per[dominant][0]
    dom_flops = 2 * w.M * w.h * w.f  # each GEMM of the block is 2*M*h*f
    peaks = _peaks()
    sustained = ms > 2000.0
    peak = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
    achieved = dom_flops / (dom_avg_ms * 1e-3) / 1e12
    value = flops * world / (ms * 1e-3 / args.steps) / 1e12

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded randn; X~N(0,1), W~N(0,0.02^2), "
            "b~N(0,0.01^2), residual=X)",
            "config": {"workload": w.name, "M": w.M, "h": w.h, "f": w.f, "t": w.t, "reduce": args.mode,
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU, t logical shards",
                       "l2": "inputs larger than L2 (W1+W2 = 268 MB per step > 126 MB L2), no flush"},
            "pct_of_peak": {"nominal_2250": round(100 * value / world / 2250.0, 2),
                            "measured_burst": round(100 * value / world / peaks["bf16_tflops"], 2),
                            "measured_sustained": round(100 * value / world / peaks["bf16_tflops_sustained"], 2)},
            "roofline": {"kernel": dominant, "bound": "tensor", "achieved": round(achieved, 2),
                         "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                         "peak_kind": ("sustained" if sustained else "burst") + " bf16, " + peaks["source"],
                         "traffic": _traffic(dominant), "flops_per_launch": dom_flops,
                         "avg_launch_ms": dom_avg_ms},
            "kernels": {k: {"launches": v[0], "total_ms": round(v[1], 3), "share": round(v[1] / ms_traced, 4)}
                        for k, v in per.items()},
            "e2e": {"value": round(flops * world / (ms_e2e * 1e-3 / args.steps) / 1e12, 2), "unit": "TFLOP/s",
                    "h2d_bytes_per_step": X.numel() * X.element_size(),
                    "d2h_bytes_per_step": out.numel() * out.element_size()},
            "gpu_launches": launches,
            "clocks": clk.summary(),
        }
        if world == 1 and not args.no_cpu_baseline:
            c = _oracle_setup(w, dev)
            line["cpu_baseline"] = cpu_baseline(w, c)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--mode", choices=["fused", "partials"], default="fused")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    from megatron_tensor_transformer_bias_b200 import configs
    w = configs.HEADLINE
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()
