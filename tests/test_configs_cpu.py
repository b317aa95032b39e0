"""The workloads' algorithmic FLOP counts (the bench's metric) against the totals of the
workload table: two GEMMs of 2*M*h*f for the FFN block; QKV projection, causal attention
core 4*B*H*d*S(S+1)/2 and output projection for the attention sub-layer; both for the layer."""
import pytest

from megatron_tensor_transformer_bias_b200 import configs


def test_flop_totals():
    assert configs.TINY_FP32_FFN.flops == 524_288                      # 0.52 MFLOP
    assert configs.HEADLINE.flops == 549_755_813_888                   # 549.76 GFLOP
    assert round(configs.ATTN_B2_S2048.flops / 1e9, 1) == 618.5        # 412.3 + 68.7 + 137.4 GFLOP
    assert round(configs.LAYER_S2048_H8192.flops / 1e9, 1) == 3367.3   # 824.6 + 68.7 + 274.9 + 2199.0 GFLOP
    assert round(configs.ffn_sweep(2048, 8).flops / 1e9, 1) == 274.9   # 16*M*h^2 at h = 2048
    assert round(configs.ffn_sweep(22528, 1).flops / 1e12, 2) == 33.26


def test_attention_core_counts_causal_pairs():
    w = configs.ATTN_B2_S2048
    dense = configs.AttnWorkload("dense", w.B, w.S, w.h, w.H, w.d, w.t, causal=False)
    core = lambda x: x.flops - 2 * x.M * x.h * 3 * x.H * x.d - 2 * x.M * x.H * x.d * x.h
    assert core(dense) == 4 * w.B * w.H * w.d * w.S * w.S                # 137.4 GFLOP if counted dense
    assert core(w) * 2 == core(dense) + 4 * w.B * w.H * w.d * w.S        # S(S+1)/2 visible pairs


@pytest.mark.parametrize("t", configs.FFN_SHARD_COUNTS)
def test_headline_shapes_shard_evenly(t):
    w = configs.ffn_2048x4096x16384(t)
    assert w.f % t == 0 and (w.f // t) % 64 == 0 and w.h % 64 == 0 and w.M == w.batch * w.seq
