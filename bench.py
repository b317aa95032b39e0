"""Throughput of the column->row tensor-parallel block on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload all|ffn|bwd|attn|layer|sweep|fp32] [--t T] [--h H|all]
                    [--mode fused|partials] [--no-cpu-baseline] [--no-sustained]

Default (``--workload all``): one JSON line per workload, the headline last --
the tiny fp32 FFN block, the attention sub-layer, the pre-LN layer, the FFN
hidden-size sweep at h = 22528 for t = 1 and 8, the FFN block's backward pass,
the FFN block with the partials reduction, and finally the headline: one
forward of the FFN block --
column-parallel GEMM + bias + exact GeLU, row-parallel GEMM, on-device reduction
of the t logical shards + bias + residual -- at M=2048 tokens (batch 4 x seq
512), h=4096, f=16384, t=4, bf16 with fp32 accumulation, seeded synthetic
inputs.  Metric: TFLOP/s with the algorithmic count (the GEMMs, 2*M*K*N each,
and causal attention 4*B*H*d*S(S+1)/2) per step.

Under torchrun each rank runs an independent replica on its own GPU (its own
token batch, no data-path collective); the value is the total work over all
ranks divided by the slowest rank's device time.

``--impl reference`` times the fp64 CPU oracle instead (rank 0 only), on a
bounded sample of token rows per step of the same workloads.
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
DATA = "synthetic (seeded randn; X~N(0,1), W~N(0,0.02^2), b~N(0,0.01^2), residual=X)"


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            p = json.load(fh)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]),
                "sm_max_mhz": p.get("sm_max_mhz", 1965.0), "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0,
                "source": "fallback"}


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
    "gemm_bwd_recompute": ["tp_gemm.cu"] + _SHARED_SOURCES,
    "gemm_bwd_dz": ["tp_gemm.cu"] + _SHARED_SOURCES,
    "gemm_bwd_dw2": ["tp_gemm.cu"] + _SHARED_SOURCES,
    "gemm_bwd_dw1": ["tp_gemm.cu"] + _SHARED_SOURCES,
    "gemm_bwd_dx": ["tp_gemm.cu"] + _SHARED_SOURCES,
    "colsum": ["tp_simt.cu"] + _SHARED_SOURCES,
    "gemm_attn_bwd_dwo": ["tp_gemm.cu"] + _SHARED_SOURCES,
    "gemm_attn_bwd_do": ["tp_gemm.cu"] + _SHARED_SOURCES,
    "gemm_attn_bwd_dwqkv": ["tp_gemm.cu"] + _SHARED_SOURCES,
    "gemm_attn_bwd_dx": ["tp_gemm.cu"] + _SHARED_SOURCES,
    "attn_bwd_rowdot": ["tp_attention_bwd.cu"] + _SHARED_SOURCES,
    "attn_bwd_dkdv": ["tp_attention_bwd.cu"] + _SHARED_SOURCES,
    "attn_bwd_dq": ["tp_attention_bwd.cu"] + _SHARED_SOURCES,
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


# ---------------------------------------------------------------- host facts
def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max(i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas")
    except Exception:
        return os.cpu_count()


def _cpu_model():
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except Exception:
        pass
    return None


def _host():
    return {"cores": _blas_threads(), "host_cpus": os.cpu_count(), "cpu_model": _cpu_model()}


def _to64(t):
    import torch
    return t.detach().to("cpu", torch.float64).numpy()


# ---------------------------------------------------------------- workloads
class Workload:
    """One step of a workload: `step(X_dev, out_dev, stream)` runs it through the C ABI.

    `oracle_setup(dev)` builds the host-side state of the oracle (fp64 copies of the
    inputs, or chunk sources for the largest sizes); `oracle_rows(state, rng, n)` runs
    the oracle as it stands on a sample of about n output rows and returns the
    algorithmic FLOPs that sample stands for (rows / M of the workload's count)."""
    name = ""
    flops = 0
    dtype = "bf16"
    kernel_amount = {}   # kernel name -> (bound, algorithmic amount per launch, unit)
    ref_rows = 8         # token rows per step of the reference arm

    def config(self):
        return {"workload": self.name}

    def metric(self):
        return f"TFLOP/s, {self.name}, 1 B200"


class FFN(Workload):
    def __init__(self, w, mode, w2_fp16=False, headline=False):
        self.w, self.mode, self.w2_fp16, self.headline = w, mode, w2_fp16, headline
        # the fp32 block always sums fp32 partials; its name carries no mode
        self.name = w.name + ("" if mode == "fused" or w.dtype == "fp32" else "_partials") + \
            ("_w2fp16" if w2_fp16 else "")
        self.flops = w.flops
        self.dtype = "bf16" if w.dtype == "bf16" else "f32"
        if w.dtype == "bf16" and w2_fp16:
            self.dtype = "bf16 (fp16 act(Z))"
        M, h, f, t = w.M, w.h, w.f, w.t
        self.kernel_amount = {
            "gemm_column_act": ("tensor", 2 * M * h * f, "FLOP"),
            "gemm_row_fused_reduce": ("tensor", 2 * M * f * h, "FLOP"),
            "gemm_row_partials": ("tensor", 2 * M * f * h, "FLOP"),
            "reduce_partials": ("hbm", (4 * t + 2 + 2) * M * h + 2 * h, "B"),
            # fp32 workload: FFMA on the CUDA cores (2 FLOP per FMA)
            "f32_col_gemm": ("alu", 2 * M * h * f, "FLOP"),
            "f32_row_gemm": ("alu", 2 * M * f * h, "FLOP"),
        }

    def metric(self):
        return METRIC if self.headline else super().metric()

    def setup(self, dev, rank):
        import torch
        from megatron_tensor_transformer_bias_b200 import inputs
        from megatron_tensor_transformer_bias_b200 import tpblock as tb
        w = self.w
        p = inputs.ffn_inputs(w.M, w.h, w.f, w.dtype, seed=0, device=dev)
        if rank:  # each replica runs its own token batch (same weights)
            g = torch.Generator(device=dev).manual_seed(7919 * rank)
            p["X"] = torch.randn(w.M, w.h, generator=g, device=dev).to(p["X"].dtype)
        self.p = p
        W2 = inputs.as_fp16(p["W2"]) if self.w2_fp16 else p["W2"]
        self.W1 = tb.shard_columns(p["W1"], w.t)
        self.W2 = tb.shard_rows(W2, w.t)
        self.b1 = tb.shard_vector(p["b1"], w.t)
        self.b2 = p["b2"]
        dt = tb.TP_FP32 if w.dtype == "fp32" else tb.TP_BF16
        self.ws = tb.workspace(tb.tp_ffn_workspace_bytes(w.M, w.h, w.f, w.t, dt, tb.MODES[self.mode]), dev)
        self.tb = tb
        return p["X"]

    def step(self, X, out, stream):
        self.tb.tp_ffn_forward(X, self.W1, self.b1, self.W2, self.b2, X, out, mode=self.mode, ws=self.ws,
                               stream=stream)

    def config(self):
        w = self.w
        c = {"workload": self.name, "M": w.M, "h": w.h, "f": w.f, "t": w.t, "reduce": self.mode,
             "dtype": w.dtype}
        if w.dtype == "bf16":
            c["w2"] = "fp16 copy of the bf16 W2 (act(Z) in fp16)" if self.w2_fp16 else "bf16"
        return c

    # -------- oracle
    def oracle_setup(self, src):
        """src: dict of input tensors (any device); W1/W2 stay 16-bit on the host and
        are converted to fp64 chunk by chunk when they are large."""
        host = {k: v.detach().to("cpu") for k, v in src.items()}
        big = self.w.h * self.w.f > (1 << 28)
        st = {"X": _to64(host["X"]), "b1": _to64(host["b1"]), "b2": _to64(host["b2"]), "big": big}
        if big:
            st["W1"], st["W2"] = host["W1"], host["W2"]
        else:
            st["W1"], st["W2"] = _to64(host["W1"]), _to64(host["W2"])
        return st

    def oracle_rows(self, st, rng, n):
        import numpy as np
        import oracle
        w = self.w
        rows = np.sort(rng.choice(w.M, min(n, w.M), replace=False))
        X = st["X"][rows]
        if not st["big"]:
            oracle.ffn_forward(X, st["W1"], st["b1"], st["W2"], st["b2"], X)
        else:
            chunks = 16
            k = w.f // chunks

            def shards():
                for i in range(chunks):
                    c = slice(i * k, (i + 1) * k)
                    yield _to64(st["W1"][:, c]), st["b1"][c], _to64(st["W2"][c, :])

            oracle.ffn_forward_sharded(X, shards(), st["b2"], X)
        return len(rows), self.flops * len(rows) / w.M


class FFNBwd(Workload):
    """One backward pass of the FFN block (tp_ffn_backward): the input gradient dX and the
    weight and bias gradients for an upstream gradient dY.  FLOPs: the model count
    8*M*h*f (dA, dW2, dW1 and dX GEMMs); the call also recomputes step 1 (2*M*h*f more,
    reported as executed_flops_per_step).  The per-step input is X and dY, stacked."""
    ref_rows = 8

    def __init__(self, w):
        self.w = w
        self.name = "ffn_bwd_" + w.name[len("ffn_"):]
        self.flops = 2 * w.flops
        M, h, f, t = w.M, w.h, w.f, w.t
        self.kernel_amount = {k: ("tensor", 2 * M * h * f, "FLOP") for k in
                              ("gemm_bwd_recompute", "gemm_bwd_dz", "gemm_bwd_dw2", "gemm_bwd_dw1", "gemm_bwd_dx")}
        # Each step traces two colsum launches, db1 (over dZ) and db2 (over dY); their bytes,
        # M*f*2 + M*h*2 in all, are spread over the two.
        self.kernel_amount["colsum"] = ("hbm", (M * f * 2 + M * h * 2) // 2, "B")

    def setup(self, dev, rank):
        import torch
        from megatron_tensor_transformer_bias_b200 import inputs
        from megatron_tensor_transformer_bias_b200 import tpblock as tb
        w = self.w
        p = inputs.ffn_inputs(w.M, w.h, w.f, "bf16", seed=0, device=dev)
        g = torch.Generator(device=dev).manual_seed(9000 + 7919 * rank)
        p["dY"] = torch.randn(w.M, w.h, generator=g, device=dev).to(torch.bfloat16)
        self.p = p
        self.W1 = tb.shard_columns(p["W1"], w.t)
        self.W2 = tb.shard_rows(p["W2"], w.t)
        self.b1 = tb.shard_vector(p["b1"], w.t)
        self.dW1 = torch.empty(w.h, w.f, dtype=torch.float32, device=dev)
        self.dW2 = torch.empty(w.f, w.h, dtype=torch.float32, device=dev)
        self.db1 = torch.empty(w.f, dtype=torch.float32, device=dev)
        self.db2 = torch.empty(w.h, dtype=torch.float32, device=dev)
        self.ws = tb.workspace(tb.tp_ffn_backward_workspace_bytes(w.M, w.h, w.f, w.t), dev)
        self.tb = tb
        return torch.stack([p["X"], p["dY"]])

    def make_out(self, X):
        import torch
        return torch.empty_like(X[0])

    def step(self, XdY, dX, stream):
        self.tb.tp_ffn_backward(XdY[0], self.W1, self.b1, self.W2, XdY[1], dX, self.dW1, self.dW2, self.db1,
                                self.db2, dX_add=XdY[1], ws=self.ws, stream=stream)

    def config(self):
        w = self.w
        return {"workload": self.name, "M": w.M, "h": w.h, "f": w.f, "t": w.t, "dtype": "bf16",
                "gradients": "dX bf16 (+ dY, the residual path); dW1, dW2, db1, db2 fp32 kept on the device",
                "executed_flops_per_step": 10 * w.M * w.h * w.f, "e2e_io": "X and dY in, dX out"}

    def oracle_setup(self, src):
        return {k: _to64(v) for k, v in src.items()}

    def oracle_rows(self, st, rng, n):
        """The oracle's backward on n token rows (their dX rows and their share of dW, db)."""
        import numpy as np
        import oracle
        w = self.w
        rows = np.sort(rng.choice(w.M, min(n, w.M), replace=False))
        oracle.ffn_backward(st["X"][rows], st["W1"], st["b1"], st["W2"], st["dY"][rows])
        return len(rows), self.flops * len(rows) / w.M


class Attn(Workload):
    ref_rows = 8

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
            "gemm_row_partials": ("tensor", 2 * M * H * d * h, "FLOP"),
        }

    def setup(self, dev, rank):
        from megatron_tensor_transformer_bias_b200 import inputs
        from megatron_tensor_transformer_bias_b200 import tpblock as tb
        w = self.w
        a = inputs.attn_inputs(w.B, w.S, w.h, w.H, w.d, seed=rank, device=dev)
        self.p = a
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
                "causal": w.causal, "reduce": self.mode, "qkv_p_dtype": "fp16"}

    def oracle_setup(self, src):
        return {k: _to64(v) for k, v in src.items()}

    def oracle_rows(self, st, rng, n):
        """n rows of one random sequence; the oracle forms K and V for the whole sequence."""
        import numpy as np
        import oracle
        w = self.w
        b = int(rng.integers(w.B))
        rows = b * w.S + np.sort(rng.choice(w.S, min(n, w.S), replace=False))
        oracle.attn_forward(st["X"], st["Wq"], st["Wk"], st["Wv"], st["Wo"], st["bo"], st["X"], w.B, w.S, w.H,
                            w.d, w.causal, rows=rows)
        return len(rows), self.flops * len(rows) / w.M


class AttnBwd(Workload):
    """One backward pass of the attention sub-layer (tp_attn_backward).  FLOPs: the model
    count, 16*M*h*H*d for the two projections' weight and input gradients plus
    8*B*H*d*pairs for dV, dP, dQ and dK (pairs = S(S+1)/2 causal); the call also
    recomputes Q, K, V, O and the scores (reported as executed_flops_per_step).  The
    per-step input is X and dY, stacked."""
    ref_rows = 8

    def __init__(self, w):
        self.w = w
        self.name = "attn_bwd_" + w.name[len("attn_"):]
        M, h, H, d, B, S = w.M, w.h, w.H, w.d, w.B, w.S
        self.pairs = S * (S + 1) // 2 if w.causal else S * S
        self.flops = 16 * M * h * H * d + 8 * B * H * d * self.pairs
        blocks = (S + 127) // 128
        # the backward kernels work in whole 128 x 128 blocks (diagonal ones included)
        bpairs = (blocks * (blocks + 1) // 2 if w.causal else blocks * blocks) * 128 * 128
        self.kernel_amount = {
            "gemm_qkv": ("tensor", 2 * M * h * 3 * H * d, "FLOP"),
            "attention": ("tensor", 4 * B * H * d * self.pairs, "FLOP"),
            "gemm_attn_bwd_dwo": ("tensor", 2 * M * H * d * h, "FLOP"),
            "gemm_attn_bwd_do": ("tensor", 2 * M * h * H * d, "FLOP"),
            "attn_bwd_rowdot": ("hbm", M * H * d * 4, "B"),
            "attn_bwd_dkdv": ("tensor", 8 * B * H * d * bpairs, "FLOP"),
            "attn_bwd_dq": ("tensor", 6 * B * H * d * bpairs, "FLOP"),
            "gemm_attn_bwd_dwqkv": ("tensor", 2 * M * h * 3 * H * d, "FLOP"),
            "gemm_attn_bwd_dx": ("tensor", 2 * M * 3 * H * d * h, "FLOP"),
        }
        self.executed = 22 * M * h * H * d + (4 * self.pairs + 14 * bpairs) * B * H * d

    def setup(self, dev, rank):
        import torch
        from megatron_tensor_transformer_bias_b200 import inputs
        from megatron_tensor_transformer_bias_b200 import tpblock as tb
        w = self.w
        a = inputs.attn_inputs(w.B, w.S, w.h, w.H, w.d, seed=rank, device=dev)
        g = torch.Generator(device=dev).manual_seed(9100 + 7919 * rank)
        a["dY"] = torch.randn(w.M, w.h, generator=g, device=dev).to(torch.bfloat16)
        self.p = a
        self.packed = inputs.pack_qkv(a["Wq"], a["Wk"], a["Wv"], w.t, w.H, w.d)
        self.Wqkv = tb.shard_columns(self.packed, w.t)
        self.Wo = tb.shard_rows(a["Wo"], w.t)
        Hd = w.H * w.d
        self.dWqkv = torch.empty(w.h, 3 * Hd, dtype=torch.float32, device=dev)
        self.dWo = torch.empty(Hd, w.h, dtype=torch.float32, device=dev)
        self.dbqkv = torch.empty(3 * Hd, dtype=torch.float32, device=dev)
        self.dbo = torch.empty(w.h, dtype=torch.float32, device=dev)
        self.ws = tb.workspace(tb.tp_attn_backward_workspace_bytes(w.B, w.S, w.h, w.H, w.d, w.t), dev)
        self.tb = tb
        return torch.stack([a["X"], a["dY"]])

    def make_out(self, X):
        import torch
        return torch.empty_like(X[0])

    def step(self, XdY, dX, stream):
        w = self.w
        self.tb.tp_attn_backward(XdY[0], w.B, w.S, w.H, w.d, self.Wqkv, None, self.Wo, XdY[1], dX, self.dWqkv,
                                 self.dWo, self.dbqkv, self.dbo, dX_add=XdY[1], causal=w.causal, ws=self.ws,
                                 stream=stream)

    def config(self):
        w = self.w
        return {"workload": self.name, "B": w.B, "S": w.S, "h": w.h, "heads": w.H, "d": w.d, "t": w.t,
                "causal": w.causal, "dtype": "bf16",
                "gradients": "dX bf16 (+ dY, the residual path); dWqkv, dWo, dbqkv, dbo fp32 kept on the device",
                "executed_flops_per_step": self.executed, "e2e_io": "X and dY in, dX out"}

    def oracle_setup(self, src):
        return {k: _to64(v) for k, v in src.items()}

    def oracle_rows(self, st, rng, n):
        """The oracle's backward of one random head over one random sequence (its projection
        columns and rows and its attention), credited 1/(B*H) of the workload's FLOPs."""
        import numpy as np
        import oracle
        w = self.w
        b, head = int(rng.integers(w.B)), int(rng.integers(w.H))
        d = w.d
        cols = slice(head * d, (head + 1) * d)
        Wqkv_h = np.concatenate([st["Wq"][:, cols], st["Wk"][:, cols], st["Wv"][:, cols]], axis=1)
        sl = slice(b * w.S, (b + 1) * w.S)
        oracle.attn_backward_sharded(st["X"][sl], [Wqkv_h], [st["Wo"][cols]], st["dY"][sl], 1, w.S, 1, d, w.causal)
        return 1, self.flops / (w.B * w.H)


class Layer(Workload):
    ref_rows = 8

    def __init__(self, w, mode):
        self.w, self.mode = w, mode
        self.name = w.name + "_fp16w"
        self.flops = w.flops
        self.dtype = "bf16 (fp16 weight copies and intermediates)"
        M, h, H, d, B, S, f = w.M, w.h, w.H, w.d, w.B, w.S, w.f
        pairs = S * (S + 1) // 2 if w.causal else S * S
        self.kernel_amount = {
            "gemm_qkv": ("tensor", 2 * M * h * 3 * H * d, "FLOP"),
            "attention": ("tensor", 4 * B * H * d * pairs, "FLOP"),
            "gemm_column_act": ("tensor", 2 * M * h * f, "FLOP"),
            # two launches per step: the attention out-projection and the FFN row layer (mean per launch)
            "gemm_row_fused_reduce": ("tensor", (2 * M * H * d * h + 2 * M * f * h) // 2, "FLOP"),
            "gemm_row_partials": ("tensor", (2 * M * H * d * h + 2 * M * f * h) // 2, "FLOP"),
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

    def oracle_setup(self, src):
        return {k: _to64(v) for k, v in src.items()}

    def oracle_rows(self, st, rng, n):
        """n rows of one random sequence; the oracle takes LN1, K and V over the whole sequence."""
        import numpy as np
        import oracle
        w = self.w
        b = int(rng.integers(w.B))
        rows = b * w.S + np.sort(rng.choice(w.S, min(n, w.S), replace=False))
        oracle.layer_forward(st["X"], st, w.B, w.S, w.H, w.d, eps=w.eps, causal=w.causal, rows=rows)
        return len(rows), self.flops * len(rows) / w.M


def make_workloads(args):
    """The workloads of this run, the headline last."""
    from megatron_tensor_transformer_bias_b200 import configs

    def ffn(t, mode, headline=False):
        w = configs.ffn_2048x4096x16384(t) if t != 4 else configs.HEADLINE
        return FFN(w, mode, headline=headline and t == 4 and mode == "fused")

    def sweep(h, t):
        return FFN(configs.ffn_sweep(h, t), args.mode, w2_fp16=True)

    wl = args.workload
    if wl == "all":
        out = [FFN(configs.TINY_FP32_FFN, "partials"), Attn(configs.ATTN_B2_S2048, "fused"),
               Layer(configs.LAYER_S2048_H8192, "fused")]
        if args.impl != "reference":   # the oracle's sweep sample needs tens of GB of fp64 weights per step
            out += [sweep(22528, 1), sweep(22528, 8)]
        out += [FFNBwd(configs.HEADLINE), AttnBwd(configs.ATTN_B2_S2048), ffn(4, "partials"),
                ffn(4, "fused", headline=True)]
        return out
    if wl == "bwd":
        return [FFNBwd(configs.ffn_2048x4096x16384(args.t) if args.t != 4 else configs.HEADLINE)]
    if wl == "ffn":
        return [ffn(args.t, args.mode, headline=True)]
    if wl == "fp32":
        return [FFN(configs.TINY_FP32_FFN, "partials")]
    if wl == "sweep":
        hs = configs.SWEEP_HIDDEN if args.h == "all" else (int(args.h),)
        ts = configs.SWEEP_SHARDS if args.t not in configs.SWEEP_SHARDS else (args.t,)
        return [sweep(h, t) for h in hs for t in ts]
    if wl == "attn":
        return [Attn(configs.ATTN_B2_S2048, args.mode)]
    if wl == "attn_bwd":
        return [AttnBwd(configs.ATTN_B2_S2048)]
    if wl == "layer":
        return [Layer(configs.LAYER_S2048_H8192, args.mode)]
    raise ValueError(wl)


# ---------------------------------------------------------------- CPU oracle timing
def cpu_baseline(wl, st, target_s=10.0, rows_per_call=64):
    """The oracle as it stands, timed on the host cores on samples of the workload's
    token rows until about `target_s` seconds of CPU work have run (at least one call).
    FLOPs credited per call: rows / M of the workload's algorithmic count."""
    import numpy as np
    rng = np.random.default_rng(0)
    rows = calls = 0
    flops = 0.0
    t0 = time.perf_counter()
    while True:
        n, fl = wl.oracle_rows(st, rng, rows_per_call)
        rows += n
        flops += fl
        calls += 1
        dt = time.perf_counter() - t0
        if dt >= target_s:
            break
    if isinstance(wl, AttnBwd):
        sample = (f"{calls} oracle call(s) of one head over one sequence each ({calls} of the {wl.w.B * wl.w.H} "
                  f"head-sequences) of {wl.name}, fp64 numpy/OpenBLAS, {dt:.1f} s wall; credited 1/(B*H) of the "
                  f"workload's FLOPs per call")
    else:
        sample = (f"{calls} oracle call(s) of {min(rows_per_call, wl.w.M)} token rows each ({rows} rows of "
                  f"{wl.w.M}) of {wl.name}, fp64 numpy/OpenBLAS, {dt:.1f} s wall; credited rows/M of the "
                  f"workload's FLOPs")
    out = {"value": round(flops / dt / 1e12, 5), "unit": "TFLOP/s", "kind": "oracle", "sample": sample}
    out.update(_host())
    return out


def run_reference(args, wls):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import numpy as np
    from megatron_tensor_transformer_bias_b200 import inputs
    for wl in wls:
        w = wl.w
        if isinstance(wl, FFNBwd):
            import torch
            src = inputs.ffn_inputs(w.M, w.h, w.f, "bf16", seed=0, device="cpu")
            src["dY"] = torch.randn(w.M, w.h, generator=torch.Generator().manual_seed(9000)).to(torch.bfloat16)
        elif isinstance(wl, AttnBwd):
            import torch
            src = inputs.attn_inputs(w.B, w.S, w.h, w.H, w.d, seed=0, device="cpu")
            src["dY"] = torch.randn(w.M, w.h, generator=torch.Generator().manual_seed(9100)).to(torch.bfloat16)
        elif isinstance(wl, FFN):
            src = inputs.ffn_inputs(w.M, w.h, w.f, w.dtype, seed=0, device="cpu")
        elif isinstance(wl, Attn):
            src = inputs.attn_inputs(w.B, w.S, w.h, w.H, w.d, seed=0, device="cpu")
        else:
            src = inputs.layer_inputs(w.B, w.S, w.h, w.H, w.d, w.f, seed=0, device="cpu")
        st = wl.oracle_setup(src)
        del src
        rng = np.random.default_rng(1)
        n = min(wl.ref_rows, w.M)
        for _ in range(args.warmup):
            wl.oracle_rows(st, rng, n)
        flops = 0.0
        t0 = time.perf_counter()
        for _ in range(args.steps):
            flops += wl.oracle_rows(st, rng, n)[1]
        dt = time.perf_counter() - t0
        value = flops / dt / 1e12
        sample = (f"{n} of {w.M} token rows of {wl.name} per step, fp64 numpy/OpenBLAS; credited rows/M of the "
                  f"workload's FLOPs")
        if isinstance(wl, AttnBwd):
            sample = (f"one head over one sequence of {wl.name} per step, fp64 numpy/OpenBLAS; credited 1/(B*H) of "
                      f"the workload's FLOPs")
        cb = {"value": value, "unit": "TFLOP/s", "kind": "oracle", "sample": sample}
        cb.update(_host())
        line = {"metric": wl.metric(), "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": wl.config(),
                "impl": "reference", "cpu_baseline": cb,
                "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        del st


# ---------------------------------------------------------------- GPU arm
def run_ours(args, wls):
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
    try:
        tb.lib()
        for wl in wls:
            run_one(args, wl, world, rank, local, dev, dist)
            torch.cuda.empty_cache()
    finally:
        if world > 1:
            dist.destroy_process_group()


def run_one(args, wl, world, rank, local, dev, dist):
    import torch
    from megatron_tensor_transformer_bias_b200 import tpblock as tb

    def barrier():
        if world > 1:
            dist.barrier()

    X = wl.setup(dev, rank)
    out = wl.make_out(X) if hasattr(wl, "make_out") else torch.empty_like(X)
    stream = torch.cuda.current_stream()

    def step():
        wl.step(X, out, stream)

    for _ in range(args.warmup):
        step()
    if tb.tp_get_device_status(stream) != tb.TP_OK:
        raise RuntimeError(f"{wl.name}: device status after warm-up: " + tb.last_error())

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
        raise RuntimeError(f"{wl.name}: device status after timing: " + tb.last_error())

    # sustained: the same step looped for >= 2 s (under the power cap), timed the same way
    sustained = None
    if getattr(wl, "headline", False) and not args.no_sustained:
        k_s = max(args.steps, int(2.2 / max(ms * 1e-3 / args.steps, 1e-6)))
        with ClockSampler(local, period_s=0.05) as clk_s:
            ms_s = timed(lambda i: step(), k_s)
        if tb.tp_get_device_status(stream) != tb.TP_OK:
            raise RuntimeError(f"{wl.name}: device status after the sustained loop: " + tb.last_error())
        v_s = wl.flops * world / (ms_s * 1e-3 / k_s) / 1e12
        peaks = _peaks()
        sustained = {"value": round(v_s, 2), "unit": "TFLOP/s", "steps": k_s, "seconds": round(ms_s / 1e3, 3),
                     "ms_per_step": ms_s / k_s, "peak": peaks["bf16_tflops_sustained"],
                     "frac_of_sustained_peak": round(v_s / world / peaks["bf16_tflops_sustained"], 4),
                     "pct_of_nominal_2250": round(100 * v_s / world / 2250.0, 2), "clocks": clk_s.summary()}

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
    long_run = ms > 2000.0
    if bound == "hbm":
        peak, punit, achieved = peaks["hbm_gbs"], "GB/s", amount / (dom_avg_ms * 1e-3) / 1e9
        pkind = "measured copy" if peaks["source"] == "measured" else "fallback"
    elif bound == "alu":
        # fp32 FFMA on the CUDA cores: 148 SMs x 128 lanes x 2 FLOP per clock at the maximum SM clock
        peak = 148 * 128 * 2 * peaks["sm_max_mhz"] * 1e6 / 1e12
        punit, achieved = "TFLOP/s", amount / (dom_avg_ms * 1e-3) / 1e12
        pkind = "fp32 FFMA, 148 SMs x 128 lanes x 2 FLOP x max SM clock"
    else:
        peak = peaks["bf16_tflops_sustained"] if long_run else peaks["bf16_tflops"]
        punit, achieved = "TFLOP/s", amount / (dom_avg_ms * 1e-3) / 1e12
        pkind = ("sustained" if long_run else "burst") + " bf16, " + peaks["source"]
    value = wl.flops * world / (ms * 1e-3 / args.steps) / 1e12

    if rank == 0:
        line = {
            "metric": wl.metric(),
            "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": wl.dtype, "data": DATA,
            "config": dict(wl.config(), parallelism=f"replicas x{world}" if world > 1
                           else "single GPU, t logical shards",
                           l2="per-step operands exceed the 126 MB L2, no flush" if wl.flops > 1e11
                           else "operands fit in L2 (launch-bound workload)"),
            "pct_of_peak": {"nominal_2250": round(100 * value / world / 2250.0, 2),
                            "measured_burst": round(100 * value / world / peaks["bf16_tflops"], 2)},
            "roofline": {"kernel": dominant, "bound": bound, "achieved": round(achieved, 3), "peak": round(peak, 1),
                         "unit": punit, "frac": round(achieved / peak, 4), "peak_kind": pkind,
                         "traffic": _traffic(wl.name, dominant), "amount_per_launch": amount,
                         "amount_unit": unit, "avg_launch_ms": dom_avg_ms},
            "kernels": {k: {"launches": v[0], "total_ms": round(v[1], 3), "share": round(v[1] / ms_traced, 4)}
                        for k, v in per.items()},
            "e2e": {"value": round(wl.flops * world / (ms_e2e * 1e-3 / args.steps) / 1e12, 3), "unit": "TFLOP/s",
                    "h2d_bytes_per_step": X.numel() * X.element_size(),
                    "d2h_bytes_per_step": out.numel() * out.element_size(),
                    "pipeline": "H2D, compute, D2H on three streams, double-buffered"},
            "gpu_launches": launches,
            "clocks": clk.summary(),
        }
        if sustained:
            line["sustained"] = sustained
        if world == 1 and not args.no_cpu_baseline:
            st = wl.oracle_setup(wl.p)
            line["cpu_baseline"] = cpu_baseline(wl, st, target_s=args.cpu_seconds)
            del st
        print(json.dumps(line), flush=True)
    barrier()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["all", "ffn", "bwd", "attn", "attn_bwd", "layer", "sweep", "fp32"],
                    default="all")
    ap.add_argument("--t", type=int, default=4)
    ap.add_argument("--h", default="22528", help="sweep hidden size, or 'all'")
    ap.add_argument("--mode", choices=["fused", "partials"], default="fused")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-sustained", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    wls = make_workloads(args)
    if args.impl == "reference":
        run_reference(args, wls)
    else:
        run_ours(args, wls)


if __name__ == "__main__":
    main()
