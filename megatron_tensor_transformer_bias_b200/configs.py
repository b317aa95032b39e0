"""The five workloads of the column->row tensor-parallel block, by name and size.

Every workload is synthetic (there is no dataset on this path): shapes, value
distributions and shard counts only.  Names say what the workload is.

Notation (as on "Tensor Parallelism > Combining Column and Row Parallelism"):
M tokens (= batch * seq), h hidden, f FFN width, t logical shards, H heads,
d head dim.  Distributions: X ~ N(0, 1), weights ~ N(0, 0.02^2),
biases ~ N(0, 0.01^2), residual = the sub-layer input, LayerNorm gamma = 1,
beta = 0, eps = 1e-5.
"""
from dataclasses import dataclass, field
from typing import Optional, Tuple


@dataclass(frozen=True)
class FFNWorkload:
    name: str
    M: int
    h: int
    f: int
    t: int
    dtype: str = "bf16"          # "bf16" or "fp32"
    batch: Optional[int] = None  # informational split of M = batch * seq
    seq: Optional[int] = None

    @property
    def flops(self) -> int:
        """Algorithmic FLOPs of one block forward: the two GEMMs, 2*M*h*f each."""
        return 4 * self.M * self.h * self.f


@dataclass(frozen=True)
class AttnWorkload:
    name: str
    B: int
    S: int
    h: int
    H: int
    d: int
    t: int
    causal: bool = True

    @property
    def M(self) -> int:
        return self.B * self.S

    @property
    def flops(self) -> int:
        """QKV projection + causal (or dense) attention core + output projection."""
        M, h, H, d, S = self.M, self.h, self.H, self.d, self.S
        qkv = 2 * M * h * 3 * H * d
        pairs = S * (S + 1) // 2 if self.causal else S * S
        core = 4 * self.B * H * d * pairs
        out = 2 * M * H * d * h
        return qkv + core + out


@dataclass(frozen=True)
class LayerWorkload:
    name: str
    B: int
    S: int
    h: int
    H: int
    d: int
    f: int
    t: int
    causal: bool = True
    eps: float = 1e-5

    @property
    def M(self) -> int:
        return self.B * self.S

    @property
    def flops(self) -> int:
        a = AttnWorkload(self.name, self.B, self.S, self.h, self.H, self.d, self.t, self.causal)
        return a.flops + 4 * self.M * self.h * self.f


# Tiny fp32 FFN block: M=8, h=64, f=256, t=2, seed 0.
TINY_FP32_FFN = FFNWorkload("ffn_fp32_M8_h64_f256_t2", M=8, h=64, f=256, t=2, dtype="fp32")

# FFN block bf16 with fp32 accumulation: M=2048 (batch 4 x seq 512), h=4096, f=16384.
def ffn_2048x4096x16384(t: int) -> FFNWorkload:
    return FFNWorkload(f"ffn_bf16_M2048_h4096_f16384_t{t}", M=2048, h=4096, f=16384, t=t,
                       batch=4, seq=512)

FFN_SHARD_COUNTS = (1, 2, 4, 8)

# Attention sub-layer bf16: batch 2, seq 2048, h=4096, 32 heads x 128, causal, t=4.
ATTN_B2_S2048 = AttnWorkload("attn_bf16_B2_S2048_h4096_H32_d128_t4_causal",
                             B=2, S=2048, h=4096, H=32, d=128, t=4, causal=True)

# Full pre-LN transformer layer bf16: batch 1, seq 2048, h=8192, 64 heads x 128,
# f=32768, t=8, causal.
LAYER_S2048_H8192 = LayerWorkload("layer_bf16_B1_S2048_h8192_H64_d128_f32768_t8_causal",
                                  B=1, S=2048, h=8192, H=64, d=128, f=32768, t=8)

# FFN hidden-size sweep bf16: M=4096, h=2048..22528 step 2048, f=4h, t in {1, 8}.
SWEEP_HIDDEN = tuple(range(2048, 22528 + 1, 2048))
SWEEP_SHARDS = (1, 8)

def ffn_sweep(h: int, t: int) -> FFNWorkload:
    return FFNWorkload(f"ffn_bf16_M4096_h{h}_f{4*h}_t{t}", M=4096, h=h, f=4 * h, t=t)

# Headline workload: the FFN block at M=2048, h=4096, f=16384 with t=4 logical shards.
HEADLINE = ffn_2048x4096x16384(4)

# Number of token rows the oracle checks at full size.
SAMPLED_ROWS = 64
