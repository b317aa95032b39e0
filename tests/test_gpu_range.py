"""fp16 intermediates and their range: a value above 65504 (the largest fp16
number) that a kernel stores in an fp16 intermediate makes
tp_get_device_status() return TP_ERR_RANGE, without a fault, and the status is
clear again afterwards.  bf16 intermediates have fp32's range and report
nothing.  The overflowing inputs are ordinary finite tensors scaled on the host
side of the call."""
import pytest
import torch

from megatron_tensor_transformer_bias_b200 import inputs
from megatron_tensor_transformer_bias_b200 import tpblock as tb

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _ffn(inp, t, w2_fp16, scale):
    X = (inp["X"].float() * scale).to(torch.bfloat16)
    W2 = inputs.as_fp16(inp["W2"]) if w2_fp16 else inp["W2"]
    out = torch.empty_like(X)
    tb.tp_ffn_forward(X, tb.shard_columns(inp["W1"], t), tb.shard_vector(inp["b1"], t), tb.shard_rows(W2, t),
                      inp["b2"], X, out)
    return out


def test_ffn_fp16_act_overflow_is_reported_and_cleared():
    inp = inputs.ffn_inputs(256, 256, 1024, "bf16", seed=41, device=DEV)
    assert tb.tp_get_device_status() == tb.TP_OK
    _ffn(inp, 2, w2_fp16=True, scale=1.0)
    assert tb.tp_get_device_status() == tb.TP_OK            # ordinary inputs: in range
    _ffn(inp, 2, w2_fp16=True, scale=1e5)                    # max |Z| ~ 1.5e5 > 65504
    s = tb.tp_get_device_status()
    assert s == tb.TP_ERR_RANGE, tb.status_string(s)
    assert "act(Z)" in tb.last_error()
    assert tb.tp_get_device_status() == tb.TP_OK            # read-and-clear
    _ffn(inp, 2, w2_fp16=False, scale=1e5)                   # bf16 act(Z): nothing to report
    assert tb.tp_get_device_status() == tb.TP_OK


def test_attention_qkv_overflow_is_reported():
    B, S, h, H, d, t = 1, 128, 256, 2, 128, 2
    a = inputs.attn_inputs(B, S, h, H, d, seed=42, device=DEV)
    X = (a["X"].float() * 1e5).to(torch.bfloat16)
    Wqkv = tb.shard_columns(inputs.pack_qkv(a["Wq"], a["Wk"], a["Wv"], t, H, d), t)
    out = torch.empty_like(X)
    tb.tp_attn_forward(X, B, S, H, d, Wqkv, None, tb.shard_rows(a["Wo"], t), a["bo"], X, out)
    s = tb.tp_get_device_status()
    assert s == tb.TP_ERR_RANGE, tb.status_string(s)
    assert "Q/K/V" in tb.last_error()
    tb.tp_attn_forward(a["X"], B, S, H, d, Wqkv, None, tb.shard_rows(a["Wo"], t), a["bo"], a["X"], out)
    assert tb.tp_get_device_status() == tb.TP_OK


def test_layernorm_fp16_output_overflow_is_reported():
    M, h = 4, 512
    g = torch.Generator(device=DEV).manual_seed(43)
    x = torch.randn(M, h, generator=g, device=DEV).to(torch.bfloat16)
    gamma = torch.full((h,), 1e5, device=DEV).to(torch.bfloat16)     # |y| ~ 1e5 > 65504
    y = torch.empty(M, h, dtype=torch.float16, device=DEV)
    tb.tp_layernorm_forward(x, gamma, None, 1e-5, y)
    s = tb.tp_get_device_status()
    assert s == tb.TP_ERR_RANGE, tb.status_string(s)
    assert "LayerNorm" in tb.last_error()
    yb = torch.empty(M, h, dtype=torch.bfloat16, device=DEV)
    tb.tp_layernorm_forward(x, gamma, None, 1e-5, yb)                # bf16 output: in range
    assert tb.tp_get_device_status() == tb.TP_OK
