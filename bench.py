"""Throughput of the column->row tensor-parallel block on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload ffn|attn|layer|sweep] [--t T] [--h H] [--mode fused|partials]

Default step (the headline): one forward of the FFN block -- column-parallel
GEMM + bias + exact GeLU, row-parallel GEMM, on-device reduction of the t
logical shards + bias + residual -- at M=2048 tokens (batch 4 x seq 512),
h=4096, f=16384, t=4, bf16 with fp32 accumulation, seeded synthetic inputs.
Metric: TFLOP/s with the algorithmic count 4*M*h*f per step.  Other workloads
(the attention sub-layer, the pre-LN layer, the FFN hidden-size sweep) print the
same line for their own algorithmic FLOP count.

Under torchrun each rank runs an independent replica on its own GPU (its own
token batch, no data-path collective); the value is the total work over all
ranks divided by the slowest rank's device time.

``--impl reference`` times the fp64 CPU oracle instead (rank 0 only), on a
bounded sample of token rows per step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import re
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


def _code_only(src: str) -> str:
    """Source text without comments and with whitespace collapsed: what the compiler sees."""
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    return re.sub(r"\s+", " ", src).strip()


def _csrc_sha():
    """Hash of the kernel sources (comments and layout ignored) that the ncu figures are keyed on."""
    d = os.path.join(ROOT, "megatron_tensor_transformer_bias_b200", "csrc")
    h = hashlib.sha256()
    for f in sorted(os.listdir(d)):
        with open(os.path.join(d, f), encoding="utf-8") as fh:
            h.update(f.encode() + _code_only(fh.read()).encode())
    return h.hexdigest()[:16]


# The sources that define each traced launch: its kernel file, the shared device helpers
# and declarations, and the host code that builds its launch (tensor maps, grid, workspace).
_SHARED_SOURCES = ["tp_ptx.cuh", "tp_internal.h", "tp_api.cu"]
KERNEL_SOURCES = {
    "gemm_column_act": ["tp_gemm.cu"] + _SHARED_SOURCES,
    "gemm_row_fused_reduce": ["tp_gemm.cu"] + _SHARED_SOURCES,
    "gemm_row_partials": ["tp_gemm.cu"] + _SHARED_SOURCES,
    "gemm_qkv": ["tp_gemm.cu"] + _SHARED_SOURCES,
    "attention": ["tp_attention.cu"] + _SHARED_SOURCES,
    "reduce_partials": ["tp_simt.cu"] + _SHARED_SOURCES,
    "layernorm": ["tp_simt.cu"] + _SHARED_SOURCES,
}


def _kernel_sha(kernel):
    """Hash of the sources (comments and layout ignored) that define one traced launch;
    the whole source tree for a launch not listed."""
    files = KERNEL_SOURCES.get(kernel)
    if not files:
        return _csrc_sha()
    d = os.path.join(ROOT, "megatron_tensor_transformer_bias_b200", "csrc")
    h = hashlib.sha256()
    for f in sorted(files):
        with open(os.path.join(d, f), encoding="utf-8") as fh:
            h.update(f.encode() + _code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def _traffic(workload, kernel):
    """DRAM bytes per launch from the committed ncu capture, or None if the sources that
    define the kernel changed since."""
    try:
        with open(os.path.join(PROFILES, "ncu_traffic.json")) as fh:
            t = json.load(fh)
    except Exception:
        return None
    rec = t.get(f"{workload}:{kernel}")
    if not rec or rec.get("src_sha") != _kernel_sha(kernel):
        return None
    return rec["dram_bytes_per_launch"]


def max_over_ranks(value, world, dist=None, device=None):
    """The slowest rank's time (every rank calls this, in the same order)."""
    if world <= 1:
        return value
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML (read-only) in a thread."""

    def __init__(self, gpu_index, period_s=0.01):
        self.idx, self.period = gpu_index, period_s
        self.samples, self.reasons, self.max_mhz, self.power = [], set(), None, []
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
                    self.power.append(self.nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0)
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
        out = {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
               "reasons": sorted(self.reasons), "samples": len(self.samples)}
        if self.power:
            out["power_w_max"] = round(max(self.power), 1)
        return out


# ---------------------------------------------------------------- workloads
class Workload:
    """One step of a workload: `step(X_dev, out_dev)` runs it through the C ABI."""
    name = ""
    flops = 0
    kernel_amount = {}   # kernel name -> (bound, algorithmic amount per launch, unit)

    def config(self):
        return {"workload": self.name}


class FFN(Workload):
    def __init__(self, w, mode, w2_fp16=False):
        self.w, self.mode, self.w2_fp16 = w, mode, w2_fp16
        self.name = w.name + ("" if mode == "fused" else "_partials") + ("_w2fp16" if w2_fp16 else "")
        self.flops = w.flops
        M, h, f, t = w.M, w.h, w.f, w.t
        self.kernel_amount = {
            "gemm_column_act": ("tensor", 2 * M * h * f, "FLOP"),
            "gemm_row_fused_reduce": ("tensor", 2 * M * f * h, "FLOP"),
            "gemm_row_partials": ("tensor", 2 * M * f * h, "FLOP"),
            "reduce_partials": ("hbm", (4 * t + 2 + 2) * M * h + 2 * h, "B"),
        }

    def setup(self, dev, rank):
        import torch
        from megatron_tensor_transformer_bias_b200 import inputs
        from megatron_tensor_transformer_bias_b200 import tpblock as tb
        w = self.w
        p = inputs.ffn_inputs(w.M, w.h, w.f, "bf16", seed=0, device=dev)
        if rank:  # each replica runs its own token batch (same weights)
            g = torch.Generator(device=dev).manual_seed(7919 * rank)
            p["X"] = torch.randn(w.M, w.h, generator=g, device=dev).to(torch.bfloat16)
        W2 = inputs.as_fp16(p["W2"]) if self.w2_fp16 else p["W2"]
        self.W1 = tb.shard_columns(p["W1"], w.t)
        self.W2 = tb.shard_rows(W2, w.t)
        self.b1 = tb.shard_vector(p["b1"], w.t)
        self.b2 = p["b2"]
        self.ws = tb.workspace(tb.tp_ffn_workspace_bytes(w.M, w.h, w.f, w.t, tb.TP_BF16, tb.MODES[self.mode]), dev)
        self.tb = tb
        return p["X"]

    def step(self, X, out, stream):
        self.tb.tp_ffn_forward(X, self.W1, self.b1, self.W2, self.b2, X, out, mode=self.mode, ws=self.ws,
                               stream=stream)

    def config(self):
        w = self.w
        return {"workload": self.name, "M": w.M, "h": w.h, "f": w.f, "t": w.t, "reduce": self.mode,
                "w2": "fp16" if self.w2_fp16 else "bf16"}


class Attn(Workload):
    def __init__(self, w, mode):
        self.w, self.mode = w, mode
        self.name = w.name
        self.flops = w.flops
        M, h, H, d, B, S = w.M, w.h, w.H, w.d, w.B, w.S
        pairs = S * (S + 1) // 2 if w.causal else S * S
        self.kernel_amount = {
            "gemm_qkv": ("tensor", 2 * M * h * 3 * H * d, "FLOP"),
            "attention": ("tensor", 4 * B * H * d * pairs, "FLOP"),
            "gemm_row_fused_reduce": ("tensor", 2 * M * H * d * h, "FLOP"),
        }

    def setup(self, dev, rank):
        from megatron_tensor_transformer_bias_b200 import inputs
        from megatron_tensor_transformer_bias_b200 import tpblock as tb
        w = self.w
        a = inputs.attn_inputs(w.B, w.S, w.h, w.H, w.d, seed=rank, device=dev)
        self.Wqkv = tb.shard_columns(inputs.pack_qkv(a["Wq"], a["Wk"], a["Wv"], w.t, w.H, w.d), w.t)
        self.Wo = tb.shard_rows(a["Wo"], w.t)
        self.bo = a["bo"]
        self.ws = tb.workspace(tb.tp_attn_workspace_bytes(w.B, w.S, w.h, w.H, w.d, w.t, tb.MODES[self.mode]), dev)
        self.tb = tb
        return a["X"]

    def step(self, X, out, stream):
        w = self.w
        self.tb.tp_attn_forward(X, w.B, w.S, w.H, w.d, self.Wqkv, None, self.Wo, self.bo, X, out, causal=w.causal,
                                mode=self.mode, ws=self.ws, stream=stream)

    def config(self):
        w = self.w
        return {"workload": self.name, "B": w.B, "S": w.S, "h": w.h, "heads": w.H, "d": w.d, "t": w.t,
                "causal": w.causal, "reduce": self.mode}


class Layer(Workload):
    def __init__(self, w, mode):
        self.w, self.mode = w, mode
        self.name = w.name + "_fp16w"
        self.flops = w.flops
        M, h, H, d, B, S, f = w.M, w.h, w.H, w.d, w.B, w.S, w.f
        pairs = S * (S + 1) // 2 if w.causal else S * S
        self.kernel_amount = {
            "gemm_qkv": ("tensor", 2 * M * h * 3 * H * d, "FLOP"),
            "attention": ("tensor", 4 * B * H * d * pairs, "FLOP"),
            "gemm_column_act": ("tensor", 2 * M * h * f, "FLOP"),
            # two launches per step: the attention out-projection and the FFN row layer (mean per launch)
            "gemm_row_fused_reduce": ("tensor", (2 * M * H * d * h + 2 * M * f * h) // 2, "FLOP"),
            "layernorm": ("hbm", 5 * M * h, "B"),
        }

    def setup(self, dev, rank):
        from megatron_tensor_transformer_bias_b200 import inputs
        from megatron_tensor_transformer_bias_b200 import tpblock as tb
        w = self.w
        p = inputs.layer_inputs(w.B, w.S, w.h, w.H, w.d, w.f, seed=rank, device=dev)
        f16 = inputs.as_fp16
        self.p = p
        self.Wqkv = tb.shard_columns(f16(inputs.pack_qkv(p["Wq"], p["Wk"], p["Wv"], w.t, w.H, w.d)), w.t)
        self.Wo = tb.shard_rows(f16(p["Wo"]), w.t)
        self.W1 = tb.shard_columns(f16(p["W1"]), w.t)
        self.W2 = tb.shard_rows(f16(p["W2"]), w.t)
        self.b1 = tb.shard_vector(p["b1"], w.t)
        self.ws = tb.workspace(tb.tp_layer_workspace_bytes(w.B, w.S, w.h, w.H, w.d, w.f, w.t,
                                                           tb.MODES[self.mode]), dev)
        self.tb = tb
        return p["X"]

    def step(self, X, out, stream):
        w, p = self.w, self.p
        self.tb.tp_layer_forward(X, w.B, w.S, w.H, w.d, p["ln1_g"], p["ln1_b"], self.Wqkv, None, self.Wo, p["bo"],
                                 p["ln2_g"], p["ln2_b"], self.W1, self.b1, self.W2, p["b2"], out, eps=w.eps,
                                 causal=w.causal, mode=self.mode, ws=self.ws, stream=stream)

    def config(self):
        w = self.w
        return {"workload": self.name, "B": w.B, "S": w.S, "h": w.h, "heads": w.H, "d": w.d, "f": w.f, "t": w.t,
                "causal": w.causal, "reduce": self.mode, "weights": "fp16 copies of the bf16 weights"}


def make_workload(args):
    from megatron_tensor_transformer_bias_b200 import configs
    if args.workload == "ffn":
        w = configs.ffn_2048x4096x16384(args.t) if args.t != 4 else configs.HEADLINE
        return FFN(w, args.mode)
    if args.workload == "sweep":
        return FFN(configs.ffn_sweep(args.h, args.t if args.t in configs.SWEEP_SHARDS else 8), args.mode,
                   w2_fp16=True)
    if args.workload == "attn":
        return Attn(configs.ATTN_B2_S2048, args.mode)
    if args.workload == "layer":
        return Layer(configs.LAYER_S2048_H8192, args.mode)
    raise ValueError(args.workload)


# ---------------------------------------------------------------- CPU oracle timing
def _threads():
    try:
        from threadpoolctl import threadpool_info
        return max(i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas")
    except Exception:
        return os.cpu_count()


def _oracle_ffn_setup(w, device):
    import torch
    from megatron_tensor_transformer_bias_b200 import inputs
    p = inputs.ffn_inputs(w.M, w.h, w.f, "bf16", seed=0, device=device)
    return {k: v.to("cpu", dtype=torch.float64).numpy() for k, v in p.items()}


def _oracle_ffn_rows(c, rows):
    import oracle
    X = c["X"][rows]
    return oracle.ffn_forward(X, c["W1"], c["b1"], c["W2"], c["b2"], X)


def cpu_baseline(w, c, target_s=10.0):
    """The oracle as it stands, on the FFN workload's token rows, timed on the host cores.

    Repeats whole passes over the M rows (or a single pass over a subset when one pass
    would take longer) until about `target_s` seconds of CPU work have run."""
    import numpy as np
    rng = np.random.default_rng(0)
    n0 = min(64, w.M)
    t0 = time.perf_counter()
    _oracle_ffn_rows(c, np.sort(rng.choice(w.M, n0, replace=False)))
    per_row = (time.perf_counter() - t0) / n0
    n = int(min(w.M, max(n0, target_s / max(per_row, 1e-9))))
    reps = max(1, int(target_s / max(per_row * n, 1e-9)))
    rows = np.arange(w.M) if n == w.M else np.sort(rng.choice(w.M, n, replace=False))
    t0 = time.perf_counter()
    for _ in range(reps):
        _oracle_ffn_rows(c, rows)
    dt = time.perf_counter() - t0
    flops = 4 * n * w.h * w.f * reps
    return {"value": round(flops / dt / 1e12, 4), "unit": "TFLOP/s", "cores": _threads(), "kind": "oracle",
            "sample": f"{reps} pass(es) over {n} of {w.M} token rows of {w.name}, fp64 numpy/OpenBLAS, "
                      f"{dt:.1f} s wall"}


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import numpy as np
    w = wl.w if isinstance(wl, FFN) else None
    if w is None:
        print(json.dumps({"impl": "reference", "unavailable": "the CPU reference arm covers the FFN workloads"}))
        return
    c = _oracle_ffn_setup(w, "cpu")
    rng = np.random.default_rng(1)
    rows_per_step = 8
    for _ in range(args.warmup):
        _oracle_ffn_rows(c, np.sort(rng.choice(w.M, rows_per_step, replace=False)))
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _oracle_ffn_rows(c, np.sort(rng.choice(w.M, rows_per_step, replace=False)))
    dt = time.perf_counter() - t0
    value = 4 * rows_per_step * w.h * w.f * args.steps / dt / 1e12
    sample = f"{rows_per_step} of {w.M} token rows of {w.name} per step, fp64 numpy/OpenBLAS"
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": wl.config(),
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": _threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- GPU arm
def run_ours(args, wl):
    import torch
    import torch.distributed as dist

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
    X = wl.setup(dev, rank)
    out = torch.empty_like(X)
    stream = torch.cuda.current_stream()

    def step():
        wl.step(X, out, stream)

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
        for i in range(k):
            fn(i)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        return max_over_ranks(e0.elapsed_time(e1), world, dist, dev)

    # end to end through the public API: every step copies its input from pinned host
    # memory and its result back to pinned host memory.  Copies run on their own streams,
    # double-buffered, so step i's copies overlap the compute of its neighbours.
    Xh = X.cpu().pin_memory()
    outh = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    Xd = [torch.empty_like(X) for _ in range(2)]
    outd = [torch.empty_like(out) for _ in range(2)]
    s_h2d = torch.cuda.Stream()
    s_d2h = torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def step_e2e(i):
        b = i & 1
        with torch.cuda.stream(s_h2d):
            s_h2d.wait_event(ev_done[b])        # Xd[b] no longer read by step i-2
            Xd[b].copy_(Xh, non_blocking=True)
            ev_in[b].record(s_h2d)
        stream.wait_event(ev_in[b])
        stream.wait_event(ev_out[b])            # outd[b] already copied out by step i-2
        wl.step(Xd[b], outd[b], stream)
        ev_done[b].record(stream)
        with torch.cuda.stream(s_d2h):
            s_d2h.wait_event(ev_done[b])
            outh[b].copy_(outd[b], non_blocking=True)
            ev_out[b].record(s_d2h)

    with ClockSampler(local) as clk:
        ms = timed(lambda i: step(), args.steps)
        tb.tp_trace_enable(16 * args.steps + 16)
        ms_traced = timed(lambda i: step(), args.steps)
        recs = tb.tp_trace_records()
        tb.tp_trace_disable()
        for i in range(3):
            step_e2e(i)
        torch.cuda.synchronize()
        ms_e2e = timed(step_e2e, args.steps)
    if tb.tp_get_device_status(stream) != tb.TP_OK:
        raise RuntimeError("device status after timing: " + tb.last_error())

    per = {}
    for name, kms in recs:
        d = per.setdefault(name, [0, 0.0])
        d[0] += 1
        d[1] += kms
    dominant = max(per, key=lambda k: per[k][1])
    launches = sum(v[0] for v in per.values())
    dom_avg_ms = per[dominant][1] / per[dominant][0]
    bound, amount, unit = wl.kernel_amount.get(dominant, ("tensor", 0, "FLOP"))
    peaks = _peaks()
    sustained = ms > 2000.0
    if bound == "hbm":
        peak, punit, achieved = peaks["hbm_gbs"], "GB/s", amount / (dom_avg_ms * 1e-3) / 1e9
        pkind = "measured copy" if peaks["source"] == "measured" else "fallback"
    else:
        peak = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
        punit, achieved = "TFLOP/s", amount / (dom_avg_ms * 1e-3) / 1e12
        pkind = ("sustained" if sustained else "burst") + " bf16, " + peaks["source"]
    value = wl.flops * world / (ms * 1e-3 / args.steps) / 1e12

    if rank == 0:
        line = {
            "metric": METRIC if isinstance(wl, FFN) and wl.w.t == 4 and wl.w.M == 2048 and wl.w.h == 4096
            else f"TFLOP/s, {wl.name}, 1 B200",
            "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16" if not isinstance(wl, Layer) else "bf16/f16",
            "data": "synthetic (seeded randn; X~N(0,1), W~N(0,0.02^2), b~N(0,0.01^2), residual=X)",
            "config": dict(wl.config(), parallelism=f"replicas x{world}" if world > 1
                           else "single GPU, t logical shards",
                           l2="per-step operands exceed the 126 MB L2, no flush"),
            "pct_of_peak": {"nominal_2250": round(100 * value / world / 2250.0, 2),
                            "measured_burst": round(100 * value / world / peaks["bf16_tflops"], 2),
                            "measured_sustained": round(100 * value / world / peaks["bf16_tflops_sustained"], 2)},
            "roofline": {"kernel": dominant, "bound": bound, "achieved": round(achieved, 2), "peak": peak,
                         "unit": punit, "frac": round(achieved / peak, 4), "peak_kind": pkind,
                         "traffic": _traffic(wl.name, dominant), "amount_per_launch": amount,
                         "amount_unit": unit, "avg_launch_ms": dom_avg_ms},
            "kernels": {k: {"launches": v[0], "total_ms": round(v[1], 3), "share": round(v[1] / ms_traced, 4)}
                        for k, v in per.items()},
            "e2e": {"value": round(wl.flops * world / (ms_e2e * 1e-3 / args.steps) / 1e12, 2), "unit": "TFLOP/s",
                    "h2d_bytes_per_step": X.numel() * X.element_size(),
                    "d2h_bytes_per_step": out.numel() * out.element_size(),
                    "pipeline": "H2D, compute, D2H on three streams, double-buffered"},
            "gpu_launches": launches,
            "clocks": clk.summary(),
        }
        if world == 1 and not args.no_cpu_baseline and isinstance(wl, FFN):
            c = _oracle_ffn_setup(wl.w, dev)
            line["cpu_baseline"] = cpu_baseline(wl.w, c)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["ffn", "attn", "layer", "sweep"], default="ffn")
    ap.add_argument("--t", type=int, default=4)
    ap.add_argument("--h", type=int, default=22528)
    ap.add_argument("--mode", choices=["fused", "partials"], default="fused")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    wl = make_workload(args)
    if args.impl == "reference":
        run_reference(args, wl)
    else:
        run_ours(args, wl)


if __name__ == "__main__":
    main()
