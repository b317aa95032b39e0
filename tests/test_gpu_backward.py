"""GPU parity of the FFN block's backward pass (tp_ffn_backward) against the fp64 oracle.

Small cases compare every element of every gradient.  The full-size workload
(M=2048, h=4096, f=16384, t=4) compares sampled outputs the oracle computes one
by one: 64 rows of dX (each row's input gradient depends on its own row only),
and dW1 columns, db1 entries and dW2 rows of 64 sampled hidden units (each hidden
unit's gradients depend on that unit alone, so the oracle runs on the block
restricted to those units).  Tolerance (``tests/parity.py``, derived from the
arithmetic): relative Frobenius <= 5e-3 as for the forward pass, and per element
6 u sqrt(sum_k (a_k b_k)^2) (+ u |ref| for the bf16 dX), u = 2^-8, for the
element's sum of products sum_k a_k b_k whose rounded factor is act(Z) or dZ."""
import numpy as np
import pytest
import torch

import oracle
from megatron_tensor_transformer_bias_b200 import configs, inputs
from megatron_tensor_transformer_bias_b200 import tpblock as tb
from tests.parity import assert_grad_close, grad_scales, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _dY(M, h, seed):
    g = torch.Generator(device=DEV).manual_seed(9000 + seed)
    return torch.randn(M, h, generator=g, device=DEV).to(torch.bfloat16)


def _run_bwd(inp, dY, t, act="gelu", with_b1=True, add_dY=True):
    X = inp["X"]
    M, h = X.shape
    f = inp["W1"].shape[1]
    dX = torch.empty_like(X)
    dW1 = torch.empty(h, f, dtype=torch.float32, device=DEV)
    dW2 = torch.empty(f, h, dtype=torch.float32, device=DEV)
    db1 = torch.empty(f, dtype=torch.float32, device=DEV)
    db2 = torch.empty(h, dtype=torch.float32, device=DEV)
    for o in (dX, dW1, dW2, db1, db2):
        o.fill_(float("nan"))
    tb.tp_ffn_backward(X, tb.shard_columns(inp["W1"], t), tb.shard_vector(inp["b1"], t) if with_b1 else None,
                       tb.shard_rows(inp["W2"], t), dY, dX, dW1, dW2, db1, db2, dX_add=dY if add_dY else None,
                       act=act)
    assert tb.tp_get_device_status() == tb.TP_OK
    return {"dX": dX, "dW1": dW1, "dW2": dW2, "db1": db1, "db2": db2}


def _oracle(inp, dY, act="gelu", with_b1=True, add_dY=True):
    X = to64(inp["X"])
    g = oracle.ffn_backward(X, to64(inp["W1"]), to64(inp["b1"]) if with_b1 else None, to64(inp["W2"]), to64(dY),
                            act=act)
    if add_dY:
        g["dX"] = g["dX"] + to64(dY)
    return g


# (300, 10176, 256, 2): its dX GEMM (N = h = 10176, two blocks of rows) runs on 256 x 512 tiles;
# (1100, 256, 512, 2): the column sums' batched eight-row loads and their one-row tail both run
SMALL = [(300, 256, 1024, 4), (1, 64, 256, 2), (129, 128, 512, 1), (513, 512, 2048, 8), (64, 192, 384, 3),
         (300, 10176, 256, 2), (1100, 256, 512, 2)]


@pytest.mark.parametrize("M,h,f,t", SMALL)
@pytest.mark.parametrize("act", ["gelu", "relu"])
def test_backward_small_full(M, h, f, t, act):
    inp = inputs.ffn_inputs(M, h, f, "bf16", seed=51, device=DEV)
    dY = _dY(M, h, 51)
    got = _run_bwd(inp, dY, t, act=act)
    ref = _oracle(inp, dY, act=act)
    sc = grad_scales(inp["X"], inp["W1"], inp["b1"], inp["W2"], dY, act)
    for k in ("dX", "dW1", "dW2", "db1", "db2"):
        assert_grad_close(got[k], ref[k], sc[k], f"{k} M{M} h{h} f{f} t{t} {act}", bf16_out=k == "dX")


def test_backward_without_bias_or_residual_gradient():
    inp = inputs.ffn_inputs(200, 256, 1024, "bf16", seed=52, device=DEV)
    dY = _dY(200, 256, 52)
    got = _run_bwd(inp, dY, 2, with_b1=False, add_dY=False)
    ref = _oracle(inp, dY, with_b1=False, add_dY=False)
    sc = grad_scales(inp["X"], inp["W1"], None, inp["W2"], dY)
    for k in ("dX", "dW1", "dW2", "db1", "db2"):
        assert_grad_close(got[k], ref[k], sc[k], f"{k} no b1, no dX_add", bf16_out=k == "dX")


def test_backward_special_cases_and_determinism():
    inp = inputs.ffn_inputs(256, 256, 1024, "bf16", seed=53, device=DEV)
    dY = _dY(256, 256, 53)
    # W2 = 0: nothing flows into the column layer; dX is dX_add exactly
    z = dict(inp)
    z["W2"] = torch.zeros_like(inp["W2"])
    got = _run_bwd(z, dY, 4)
    assert torch.equal(got["dX"], dY)
    assert not got["dW1"].any() and not got["db1"].any()
    assert_grad_close(got["dW2"], _oracle(z, dY)["dW2"], grad_scales(z["X"], z["W1"], z["b1"], z["W2"], dY)["dW2"],
                      "dW2 with W2 = 0")
    # dY = 0: every gradient is zero
    got = _run_bwd(inp, torch.zeros_like(dY), 2)
    for k, v in got.items():
        assert not v.any(), k
    # bitwise repeatable
    a = _run_bwd(inp, dY, 4)
    b = _run_bwd(inp, dY, 4)
    for k in a:
        assert torch.equal(a[k], b[k]), k


def test_backward_bitwise_across_t():
    """dX sums the shards' K-slices in one accumulator in the same order for every t, and
    the weight gradients' tiles line up when f/t is a multiple of 256: the same bits."""
    inp = inputs.ffn_inputs(384, 256, 2048, "bf16", seed=54, device=DEV)
    dY = _dY(384, 256, 54)
    ref = _run_bwd(inp, dY, 1)
    for t in (2, 4, 8):
        got = _run_bwd(inp, dY, t)
        for k in ref:
            assert torch.equal(got[k], ref[k]), (t, k)


def test_backward_no_rows_zeroes_the_weight_gradients():
    h, f, t = 128, 512, 2
    inp = inputs.ffn_inputs(4, h, f, "bf16", seed=55, device=DEV)
    X = inp["X"][:0]
    dY = torch.empty(0, h, dtype=torch.bfloat16, device=DEV)
    dX = torch.empty(0, h, dtype=torch.bfloat16, device=DEV)
    dW1 = torch.full((h, f), 7.0, device=DEV)
    dW2 = torch.full((f, h), 7.0, device=DEV)
    db1 = torch.full((f,), 7.0, device=DEV)
    db2 = torch.full((h,), 7.0, device=DEV)
    tb.tp_ffn_backward(X, tb.shard_columns(inp["W1"], t), None, tb.shard_rows(inp["W2"], t), dY, dX, dW1, dW2,
                       db1, db2, ws=tb.workspace(1, DEV))
    torch.cuda.synchronize()
    for v in (dW1, dW2, db1, db2):
        assert not v.any()


@pytest.fixture(scope="module")
def bwd_full():
    w = configs.HEADLINE
    inp = inputs.ffn_inputs(w.M, w.h, w.f, "bf16", seed=0, device=DEV)
    dY = _dY(w.M, w.h, 0)
    got = _run_bwd(inp, dY, w.t)
    yield w, inp, dY, got
    del inp, got
    torch.cuda.empty_cache()


def test_backward_2048x4096x16384_t4_sampled_rows(bwd_full):
    w, inp, dY, got = bwd_full
    rows = inputs.sample_rows(w.M, configs.SAMPLED_ROWS, seq=w.seq)
    X = to64(inp["X"][rows])
    g = oracle.ffn_backward(X, to64(inp["W1"]), to64(inp["b1"]), to64(inp["W2"]), to64(dY[rows]))
    sc = grad_scales(inp["X"][rows], inp["W1"], inp["b1"], inp["W2"], dY[rows])
    assert_grad_close(got["dX"][rows], g["dX"] + to64(dY[rows]), sc["dX"], "dX sampled rows", bf16_out=True)
    assert torch.isfinite(got["dX"].float()).all()


def test_backward_2048x4096x16384_t4_sampled_hidden_units(bwd_full):
    w, inp, dY, got = bwd_full
    units = inputs.sample_rows(w.f, configs.SAMPLED_ROWS)      # 64 of the f hidden units
    X = to64(inp["X"])
    g = oracle.ffn_backward(X, to64(inp["W1"][:, units]), to64(inp["b1"][units]), to64(inp["W2"][units]), to64(dY))
    sc = grad_scales(inp["X"], inp["W1"][:, units], inp["b1"][units], inp["W2"][units], dY)
    assert_grad_close(got["dW1"][:, units], g["dW1"], sc["dW1"], "dW1 sampled columns")
    assert_grad_close(got["db1"][units], g["db1"], sc["db1"], "db1 sampled entries")
    assert_grad_close(got["dW2"][units], g["dW2"], sc["dW2"], "dW2 sampled rows")
    assert_grad_close(got["db2"], g["db2"], sc["db2"], "db2")
    for k in ("dW1", "dW2", "db1"):
        assert torch.isfinite(got[k]).all(), k


def test_backward_large_bias_reaches_the_recompute():
    """b1 ~ N(0, 0.5^2) moves every Z by about as much as X W1 does, so a bias dropped or
    added at the wrong column in the recomputation changes act'(Z) far beyond the bound."""
    inp = inputs.ffn_inputs(160, 128, 768, "bf16", seed=56, device=DEV)   # t = 3: f/t = 256
    inp["b1"] = (inp["b1"].float() * 50).to(torch.bfloat16)
    dY = _dY(160, 128, 56)
    got = _run_bwd(inp, dY, 3)
    ref = _oracle(inp, dY)
    sc = grad_scales(inp["X"], inp["W1"], inp["b1"], inp["W2"], dY)
    for k in ("dX", "dW1", "dW2", "db1", "db2"):
        assert_grad_close(got[k], ref[k], sc[k], f"{k} large b1", bf16_out=k == "dX")
    # and the same block without its bias differs from it by far more than the tolerance
    ref0 = _oracle(inp, dY, with_b1=False)
    assert np.linalg.norm(ref0["dW1"] - ref["dW1"]) > 0.1 * np.linalg.norm(ref["dW1"])
