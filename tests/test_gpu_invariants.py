"""Invariants of the method checked on the GPU path itself (through the C ABI), each
against a closed form computed here in fp64 rather than against the oracle:
- attention with Q = 0: every visible key has the same score, so each query's output
  is the prefix mean of V (causal);
- attention with V = 1: the softmax rows sum to one, so O = 1;
- LayerNorm: output rows have mean 0 and mean square var / (var + eps), and LN(x + c) = LN(x);
- FFN: t-fold duplicated shards with W2 halved give the unsharded block's output."""
import numpy as np
import pytest
import torch

import oracle
from megatron_tensor_transformer_bias_b200 import inputs
from megatron_tensor_transformer_bias_b200 import tpblock as tb
from tests.parity import assert_bf16_close, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _attn(a, B, S, H, d, t, bqkv=None):
    Wqkv = tb.shard_columns(inputs.pack_qkv(a["Wq"], a["Wk"], a["Wv"], t, H, d), t)
    out = torch.empty_like(a["X"])
    tb.tp_attn_forward(a["X"], B, S, H, d, Wqkv, bqkv, tb.shard_rows(a["Wo"], t), a["bo"], a["X"], out,
                       causal=True)
    assert tb.tp_get_device_status() == tb.TP_OK
    return to64(out)


@pytest.mark.parametrize("B,S,H,t", [(2, 300, 4, 2), (1, 129, 2, 1)])
def test_attention_zero_queries_give_prefix_means(B, S, H, t):
    d, h = 128, 256
    a = inputs.attn_inputs(B, S, h, H, d, seed=31, device=DEV)
    a["Wq"] = torch.zeros_like(a["Wq"])
    got = _attn(a, B, S, H, d, t)
    X, Wv, Wo, bo = to64(a["X"]), to64(a["Wv"]), to64(a["Wo"]), to64(a["bo"])
    V = (X @ Wv).reshape(B, S, H * d)
    prefix = np.cumsum(V, axis=1) / np.arange(1, S + 1)[None, :, None]
    want = prefix.reshape(B * S, H * d) @ Wo + bo + X
    assert_bf16_close(torch.from_numpy(got), want, "Q = 0: prefix means of V")


def test_attention_unit_values_give_row_sums_of_one():
    B, S, H, t, d, h = 2, 200, 4, 2, 128, 256
    a = inputs.attn_inputs(B, S, h, H, d, seed=32, device=DEV)
    a["Wv"] = torch.zeros_like(a["Wv"])
    Hg = H // t
    bias = torch.zeros(3 * Hg * d, dtype=torch.bfloat16, device=DEV)
    bias[2 * Hg * d:] = 1.0                                   # V = 1 for every token and head
    got = _attn(a, B, S, H, d, t, bqkv=[bias] * t)
    X, Wo, bo = to64(a["X"]), to64(a["Wo"]), to64(a["bo"])
    want = np.ones((B * S, H * d)) @ Wo + bo + X              # O = 1: softmax rows sum to one
    assert_bf16_close(torch.from_numpy(got), want, "V = 1: O = 1")


def test_layernorm_moments_and_shift_invariance():
    M, h, eps = 64, 4096, 1e-5
    g = torch.Generator(device=DEV).manual_seed(33)
    x = torch.randn(M, h, generator=g, device=DEV) * 2 + 0.5
    y = torch.empty(M, h, dtype=torch.float16, device=DEV)
    tb.tp_layernorm_forward(x, None, None, eps, y)
    yy, xx = to64(y), to64(x)
    var = xx.var(axis=1)
    assert np.all(np.abs(yy.mean(axis=1)) < 2e-4)
    np.testing.assert_allclose((yy ** 2).mean(axis=1), var / (var + eps), rtol=2e-3)
    y2 = torch.empty_like(y)
    tb.tp_layernorm_forward(x + 4.0, None, None, eps, y2)     # fp32 input: x + 4 is exact to ~2^-21
    assert np.all(np.abs(to64(y2) - yy) <= 2.0 ** -10 * np.abs(yy) + 2e-3)


@pytest.mark.parametrize("mode", ["fused", "partials"])
def test_ffn_duplicated_shards_with_halved_w2(mode):
    M, h, f = 256, 256, 1024
    p = inputs.ffn_inputs(M, h, f, "bf16", seed=34, device=DEV)
    base = torch.empty_like(p["X"])
    tb.tp_ffn_forward(p["X"], [p["W1"]], [p["b1"]], [p["W2"]], p["b2"], p["X"], base, mode=mode)
    half = (p["W2"].float() * 0.5).to(torch.bfloat16)         # exact: a power of two
    dup = torch.empty_like(base)
    tb.tp_ffn_forward(p["X"], [p["W1"], p["W1"]], [p["b1"], p["b1"]], [half, half], p["b2"], p["X"], dup, mode=mode)
    assert tb.tp_get_device_status() == tb.TP_OK
    a, b = to64(dup), to64(base)
    assert np.all(np.abs(a - b) <= 2.0 ** -7 * np.abs(b) + 1e-6)  # only the fp32 summation order differs
    ref = oracle.ffn_forward(to64(p["X"]), to64(p["W1"]), to64(p["b1"]), to64(p["W2"]), to64(p["b2"]),
                             to64(p["X"]))
    assert_bf16_close(dup, ref, f"duplicated shards {mode}")
