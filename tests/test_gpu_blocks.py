"""GPU unit tests of the building blocks: LayerNorm, the fixed-order reduce, the
bounded-wait status path and the launch trace."""
import os

import numpy as np
import pytest
import torch

import oracle
from megatron_tensor_transformer_bias_b200 import tpblock as tb
from tests.parity import assert_bf16_close, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"


# h <= 2048, <= 4096 and <= 8192 take the register-resident kernel with 1, 2 and 4 chunks of
# 8 per thread (5000: some threads hold a third chunk, none a fourth); above 8192 the row is
# cached in shared memory.
@pytest.mark.parametrize("M,h", [(1, 8), (37, 256), (3, 4000), (7, 5000), (2048, 8192), (2, 8200), (5, 22528)])
@pytest.mark.parametrize("in_dtype", [torch.bfloat16, torch.float32])
def test_layernorm(M, h, in_dtype):
    g = torch.Generator(device=DEV).manual_seed(M * 7 + h)
    x = (torch.randn(M, h, generator=g, device=DEV) * 3 + 1).to(in_dtype)
    gamma = (1 + 0.1 * torch.randn(h, generator=g, device=DEV)).to(torch.bfloat16)
    beta = (0.1 * torch.randn(h, generator=g, device=DEV)).to(torch.bfloat16)
    y = torch.empty(M, h, dtype=torch.bfloat16, device=DEV)
    tb.tp_layernorm_forward(x, gamma, beta, 1e-5, y)
    assert_bf16_close(y, oracle.layernorm(to64(x), to64(gamma), to64(beta), 1e-5), f"LN {M}x{h}")
    y2 = torch.empty(M, h, dtype=torch.float16, device=DEV)
    tb.tp_layernorm_forward(x, None, None, 1e-5, y2)
    assert_bf16_close(y2, oracle.layernorm(to64(x), None, None, 1e-5), f"LN plain fp16 out {M}x{h}")


@pytest.mark.parametrize("t", [1, 2, 4, 8])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_reduce_partials(t, dtype):
    M, h = 333, 4096
    g = torch.Generator(device=DEV).manual_seed(t)
    P = torch.randn(t, M, h, generator=g, device=DEV)
    bias = torch.randn(h, generator=g, device=DEV).to(dtype)
    R = torch.randn(M, h, generator=g, device=DEV).to(dtype)
    out = torch.empty(M, h, dtype=dtype, device=DEV)
    tb.tp_reduce_partials(P, bias, R, out)
    ref = oracle.reduce_partials([to64(p) for p in P], to64(bias), to64(R))
    if dtype == torch.float32:
        np.testing.assert_allclose(to64(out), ref, rtol=1e-6, atol=1e-5)
        # fixed order 0..t-1 in fp32, then bias, then residual: bit-exact against the same order in torch
        acc = P[0].clone()
        for i in range(1, t):
            acc += P[i]
        acc += bias
        acc += R
        assert torch.equal(out, acc)
    else:
        assert_bf16_close(out, ref, f"reduce bf16 t{t}")


def test_bounded_wait_reports_timeout_and_context_survives():
    assert tb.tp_get_device_status() == tb.TP_OK
    tb.tp_selftest_bounded_wait(5_000_000)  # 5 ms
    assert tb.tp_get_device_status() == tb.TP_ERR_TIMEOUT
    assert "site 5" in tb.last_error()
    # the status word was cleared and the context still works
    assert tb.tp_get_device_status() == tb.TP_OK
    x = torch.ones(4, 64, dtype=torch.bfloat16, device=DEV)
    y = torch.empty_like(x)
    tb.tp_layernorm_forward(x, None, None, 1e-5, y)
    torch.cuda.synchronize()
    assert torch.equal(y, torch.zeros_like(y))


def test_launch_trace_names_kernels():
    from megatron_tensor_transformer_bias_b200 import inputs
    inp = inputs.ffn_inputs(256, 256, 1024, "bf16", seed=1, device=DEV)
    out = torch.empty_like(inp["X"])
    tb.tp_trace_enable(64)
    try:
        tb.tp_ffn_forward(inp["X"], tb.shard_columns(inp["W1"], 2), None, tb.shard_rows(inp["W2"], 2), None,
                          None, out, mode="partials")
        torch.cuda.synchronize()
        recs = tb.tp_trace_records()
    finally:
        tb.tp_trace_disable()
    names = [n for n, _ in recs]
    # partials mode: the fixed-order reduce runs after the row GEMM (inside it with
    # TPB_REDUCE_IN_GEMM=1)
    if os.environ.get("TPB_REDUCE_IN_GEMM") == "1":
        assert names == ["gemm_column_act", "gemm_row_partials"]
    else:
        assert names == ["gemm_column_act", "gemm_row_partials", "reduce_partials"]
    assert all(ms > 0 for _, ms in recs)


def test_activation_matches_exact_gelu_and_relu():
    """The column layer's nonlinearity in fp32 against the fp64 oracle: the published erfc
    approximation it uses has fractional error < 1.2e-7; in fp32 the GeLU stays within
    4e-7 absolute (2e-5 relative in the far negative tail)."""
    g = torch.Generator(device=DEV).manual_seed(41)
    x = torch.cat([torch.linspace(-14, 14, 200001, device=DEV),
                   torch.randn(100000, generator=g, device=DEV) * 3,
                   torch.tensor([0.0, -0.0, 1.0, -1.0, 2.0, 0.5, 1e-30, -1e-30, 40.0, -40.0], device=DEV)])
    y = torch.empty_like(x)
    tb.tp_activation_forward(x, y, "gelu")
    ref = oracle.gelu(to64(x))
    err = np.abs(to64(y) - ref)
    assert (err <= 1e-6 + 3e-5 * np.abs(ref)).all(), float(err.max())
    # table values of the exact GeLU, x * Phi(x)
    yy = to64(y)[-10:]
    assert yy[0] == 0.0 and yy[1] == 0.0
    assert abs(yy[2] - 0.8413447460685429) < 2e-7 and abs(yy[3] + (1 - 0.8413447460685429)) < 2e-7
    assert abs(yy[4] - 2 * 0.9772498680518208) < 4e-7 and abs(yy[5] - 0.5 * 0.6914624612740131) < 2e-7
    assert yy[8] == 40.0 and yy[9] == 0.0
    tb.tp_activation_forward(x, y, "relu")
    assert torch.equal(y, torch.clamp(x, min=0.0))
