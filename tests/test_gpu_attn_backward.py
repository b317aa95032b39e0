"""GPU parity of the attention sub-layer's backward pass (tp_attn_backward) against the fp64 oracle.

Every element of every gradient is compared on small cases (ragged and one-token
sequences, causal and not, biases or none, t = 1, 2, 4) and on one full-length
sequence (S = 2048 with four heads).  At the full workload size (B=2, S=2048,
h=4096, 32 heads, t=4) the oracle computes two sampled heads end to end: their
rows of dWo and their columns of dWqkv and dbqkv depend on those heads alone;
dbo is checked whole.

Tolerance, from the arithmetic: the gradients are sums of products whose factors
are rounded to 16 bits on the way (Q, K, V, dO, P and dS in fp16, O and dQKV in
bf16, u = 2^-8), so relative Frobenius error <= 5e-3 (the forward pass's bar) and
per element |err| <= 8 u rms(ref) + 2 u |ref|: the rounding noise of a sum of
many products is a fraction u of its typical size, with the same 8-sigma margin
for the few-term sums at the edges of causal blocks."""
import numpy as np
import pytest
import torch

import oracle
from megatron_tensor_transformer_bias_b200 import inputs
from megatron_tensor_transformer_bias_b200 import tpblock as tb
from tests.parity import BF16_REL_FRO, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"
U = 2.0 ** -8
D_HEAD = 128


def assert_attn_grad_close(got, ref, what):
    got, ref = to64(got), to64(ref)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite GPU output"
    diff = np.abs(got - ref)
    rel_fro = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))
    assert rel_fro <= BF16_REL_FRO, f"{what}: rel Frobenius {rel_fro:.3e} > {BF16_REL_FRO}"
    rms = float(np.sqrt(np.mean(ref ** 2)))
    bound = 8 * U * rms + 2 * U * np.abs(ref) + 1e-30
    worst = float((diff / bound).max())
    assert worst <= 1.0, f"{what}: element error {worst:.2f}x the bound (max |err| {diff.max():.3e}, rms {rms:.3e})"
    return rel_fro


def _case(B, S, h, H, t, seed, with_bias):
    a = inputs.attn_inputs(B, S, h, H, D_HEAD, seed=seed, device=DEV)
    packed = inputs.pack_qkv(a["Wq"], a["Wk"], a["Wv"], t, H, D_HEAD)
    g = torch.Generator(device=DEV).manual_seed(700 + seed)
    bqkv = (torch.randn(3 * H * D_HEAD, generator=g, device=DEV) * 0.01).to(torch.bfloat16) if with_bias else None
    dY = torch.randn(B * S, h, generator=g, device=DEV).to(torch.bfloat16)
    return a, packed, bqkv, dY


def _run(a, packed, bqkv, dY, B, S, H, t, causal, add_dY=True):
    X = a["X"]
    h = X.shape[1]
    Hd = H * D_HEAD
    dX = torch.full_like(X, float("nan"))
    dWqkv = torch.full((h, 3 * Hd), float("nan"), dtype=torch.float32, device=DEV)
    dWo = torch.full((Hd, h), float("nan"), dtype=torch.float32, device=DEV)
    dbqkv = torch.full((3 * Hd,), float("nan"), dtype=torch.float32, device=DEV)
    dbo = torch.full((h,), float("nan"), dtype=torch.float32, device=DEV)
    tb.tp_attn_backward(X, B, S, H, D_HEAD, tb.shard_columns(packed, t),
                        tb.shard_vector(bqkv, t) if bqkv is not None else None, tb.shard_rows(a["Wo"], t), dY, dX,
                        dWqkv, dWo, dbqkv, dbo, dX_add=dY if add_dY else None, causal=causal)
    assert tb.tp_get_device_status() == tb.TP_OK, tb.last_error()
    return {"dX": dX, "dWqkv": dWqkv, "dWo": dWo, "dbqkv": dbqkv, "dbo": dbo}


def _oracle(a, packed, bqkv, dY, B, S, H, t, causal, add_dY=True):
    Hg = H // t
    n3 = 3 * Hg * D_HEAD
    P = to64(packed)
    Wqkv = [P[:, i * n3:(i + 1) * n3] for i in range(t)]
    Wo = [to64(a["Wo"])[i * Hg * D_HEAD:(i + 1) * Hg * D_HEAD] for i in range(t)]
    bs = None if bqkv is None else [to64(bqkv)[i * n3:(i + 1) * n3] for i in range(t)]
    dX, dWqkv, dbqkv, dWo, dbo = oracle.attn_backward_sharded(to64(a["X"]), Wqkv, Wo, to64(dY), B, S, Hg, D_HEAD,
                                                              causal, bqkv_shards=bs)
    if add_dY:
        dX = dX + to64(dY)
    return {"dX": dX, "dWqkv": np.concatenate(dWqkv, axis=1), "dWo": np.concatenate(dWo, axis=0),
            "dbqkv": np.concatenate(dbqkv), "dbo": dbo}


SMALL = [(1, 128, 256, 2, 2), (2, 200, 256, 2, 1), (1, 384, 512, 4, 2), (1, 1, 256, 2, 2), (1, 700, 256, 2, 2),
         (2, 129, 512, 4, 4)]


@pytest.mark.parametrize("B,S,h,H,t", SMALL)
@pytest.mark.parametrize("causal", [True, False])
def test_attn_backward_small_full(B, S, h, H, t, causal):
    a, packed, bqkv, dY = _case(B, S, h, H, t, seed=61 + S, with_bias=True)
    got = _run(a, packed, bqkv, dY, B, S, H, t, causal)
    ref = _oracle(a, packed, bqkv, dY, B, S, H, t, causal)
    for k in ("dX", "dWqkv", "dWo", "dbqkv", "dbo"):
        assert_attn_grad_close(got[k], ref[k], f"{k} B{B} S{S} h{h} H{H} t{t} causal={causal}")


def test_attn_backward_no_bias_no_residual_gradient():
    B, S, h, H, t = 1, 256, 256, 2, 2
    a, packed, _, dY = _case(B, S, h, H, t, seed=62, with_bias=False)
    got = _run(a, packed, None, dY, B, S, H, t, True, add_dY=False)
    ref = _oracle(a, packed, None, dY, B, S, H, t, True, add_dY=False)
    for k in ("dX", "dWqkv", "dWo", "dbqkv", "dbo"):
        assert_attn_grad_close(got[k], ref[k], f"{k} no bias, no dX_add")


def test_attn_backward_full_length_sequence():
    """S = 2048 (16 query and key blocks, the workload's sequence length), four heads."""
    B, S, h, H, t = 1, 2048, 512, 4, 2
    a, packed, bqkv, dY = _case(B, S, h, H, t, seed=63, with_bias=True)
    got = _run(a, packed, bqkv, dY, B, S, H, t, True)
    ref = _oracle(a, packed, bqkv, dY, B, S, H, t, True)
    for k in ("dX", "dWqkv", "dWo", "dbqkv", "dbo"):
        assert_attn_grad_close(got[k], ref[k], f"{k} S=2048")


def test_attn_backward_deterministic_and_t_invariant():
    """Fixed-order sums: two calls give the same bits; the per-head gradients do not depend on
    how the heads are grouped, so dWo, dWqkv's per-head blocks and dbo agree across t."""
    B, S, h, H = 1, 384, 512, 4
    outs = {}
    for t in (1, 2, 4):
        a, packed, bqkv, dY = _case(B, S, h, H, t, seed=64, with_bias=False)
        r1 = _run(a, packed, None, dY, B, S, H, t, True)
        r2 = _run(a, packed, None, dY, B, S, H, t, True)
        for k in r1:
            assert torch.equal(r1[k], r2[k]), f"{k} t={t} not bitwise repeatable"
        outs[t] = r1
    for t in (2, 4):
        assert torch.equal(outs[t]["dWo"], outs[1]["dWo"]), f"dWo differs between t=1 and t={t}"
        assert torch.equal(outs[t]["dbo"], outs[1]["dbo"]), f"dbo differs between t=1 and t={t}"


def test_attn_backward_no_tokens_zeroes_gradients():
    h, H, t = 256, 2, 2
    Hd = H * D_HEAD
    a = inputs.attn_inputs(1, 1, h, H, D_HEAD, seed=65, device=DEV)
    packed = inputs.pack_qkv(a["Wq"], a["Wk"], a["Wv"], t, H, D_HEAD)
    dWqkv = torch.full((h, 3 * Hd), 7.0, device=DEV)
    dWo = torch.full((Hd, h), 7.0, device=DEV)
    dbqkv = torch.full((3 * Hd,), 7.0, device=DEV)
    dbo = torch.full((h,), 7.0, device=DEV)
    ws = tb.workspace(tb.tp_attn_backward_workspace_bytes(1, 1, h, H, D_HEAD, t), DEV)
    empty = torch.empty(0, h, dtype=torch.bfloat16, device=DEV)
    tb._check(tb.lib().tp_attn_backward(None, 0, 1, h, H, D_HEAD, t, tb._shards(tb.shard_columns(packed, t)), None,
                                        tb._shards(tb.shard_rows(a["Wo"], t)), None, None, 1, None,
                                        tb._ptr(dWqkv), tb._ptr(dbqkv), tb._ptr(dWo), tb._ptr(dbo), tb._ptr(ws),
                                        ws.numel(), None))
    torch.cuda.synchronize()
    for x in (dWqkv, dWo, dbqkv, dbo):
        assert not torch.any(x)
    del empty


@pytest.fixture(scope="module")
def attn_bwd_full():
    B, S, h, H, t = 2, 2048, 4096, 32, 4
    a, packed, bqkv, dY = _case(B, S, h, H, t, seed=66, with_bias=False)
    got = _run(a, packed, None, dY, B, S, H, t, True)
    return B, S, h, H, t, a, packed, dY, got


@pytest.mark.parametrize("head", [0, 21])
def test_attn_backward_full_size_sampled_heads(attn_bwd_full, head):
    """Workload size: one head's rows of dWo and columns of dWqkv / dbqkv (they depend on
    that head alone), computed by the oracle for that head over both sequences; dbo whole."""
    B, S, h, H, t, a, packed, dY, got = attn_bwd_full
    d = D_HEAD
    Hg = H // t
    g, hl = head // Hg, head % Hg
    n3 = 3 * Hg * d
    cols = [g * n3 + part * Hg * d + hl * d + e for part in range(3) for e in range(d)]
    P = to64(packed)
    Wqkv_h = P[:, cols]                                    # [h, 3d]: this head's [q | k | v] columns
    Wo_h = to64(a["Wo"])[head * d:(head + 1) * d]          # its rows of the output projection
    dX, dWqkv, dbqkv, dWo, dbo = oracle.attn_backward_sharded(to64(a["X"]), [Wqkv_h], [Wo_h], to64(dY), B, S, 1, d,
                                                              True)
    assert_attn_grad_close(got["dWo"][head * d:(head + 1) * d], dWo[0], f"dWo rows of head {head}")
    assert_attn_grad_close(got["dWqkv"][:, cols], dWqkv[0], f"dWqkv columns of head {head}")
    assert_attn_grad_close(got["dbqkv"][cols], dbqkv[0], f"dbqkv entries of head {head}")
    assert_attn_grad_close(got["dbo"], dbo, "dbo")
    assert torch.isfinite(got["dX"].float()).all()
