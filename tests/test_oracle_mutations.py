"""Planted mistakes in the oracle (on the CPU) must each fail a pin.

These show that the pins in ``test_oracle_pins.py`` are sensitive to the
mistakes an fp64 restatement of the block is likely to contain.
"""
import math
import types

import numpy as np
import pytest

import oracle
import oracle.tp_block as tb
from tests import test_oracle_pins as pins


def _expect_fail(check):
    with pytest.raises(AssertionError):
        check()


def test_tanh_gelu_is_caught(monkeypatch):
    # the tanh approximation written as an erf replacement: erf(u) ~ tanh(c (x + 0.044715 x^3)), x = u sqrt 2
    def erf_tanh(u):
        x = np.asarray(u) * math.sqrt(2.0)
        return np.tanh(math.sqrt(2.0 / math.pi) * (x + 0.044715 * x ** 3))
    monkeypatch.setattr(tb, "_erf", erf_tanh)
    _expect_fail(pins.check_gelu_table)


def test_wrong_attention_scale_is_caught(monkeypatch):
    fake_math = types.SimpleNamespace(sqrt=lambda x: float(x))  # 1/d instead of 1/sqrt(d)
    monkeypatch.setattr(tb, "math", fake_math)
    _expect_fail(pins.check_attention_core)


def test_off_by_one_causal_mask_is_caught(monkeypatch):
    def attention_strict(Q, K, V, causal, q_pos=None):
        Q, K, V = (np.asarray(a, float) for a in (Q, K, V))
        nq, Hn, d = Q.shape
        S = K.shape[0]
        q_pos = np.arange(nq) if q_pos is None else np.asarray(q_pos)
        keep = (np.arange(S)[None, :] < q_pos[:, None] + (0 if causal else S))
        keep[:, 0] = True  # keeps row 0 finite; the mistake is j < i elsewhere
        O = np.empty((nq, Hn, d))
        for g in range(Hn):
            s = np.where(keep, Q[:, g] @ K[:, g].T / math.sqrt(d), -np.inf)
            p = np.exp(s - s.max(1, keepdims=True))
            O[:, g] = (p / p.sum(1, keepdims=True)) @ V[:, g]
        return O
    monkeypatch.setattr(oracle, "attention_heads", attention_strict)
    monkeypatch.setattr(tb, "attention_heads", attention_strict)
    _expect_fail(pins.check_attention_core)


def test_unbiased_variance_is_caught(monkeypatch):
    def ln_unbiased(x, g, b, eps=1e-5):
        x = np.asarray(x, float)
        mu = x.mean(-1, keepdims=True)
        var = x.var(-1, ddof=1, keepdims=True)
        y = (x - mu) / np.sqrt(var + eps)
        return y * (1 if g is None else g) + (0 if b is None else b)
    monkeypatch.setattr(oracle, "layernorm", ln_unbiased)
    monkeypatch.setattr(tb, "layernorm", ln_unbiased)
    _expect_fail(pins.check_layernorm)


def test_bias_per_shard_is_caught(monkeypatch):
    real = tb.ffn_forward_sharded

    def b2_per_shard(X, shards, b2, R, act="gelu"):
        shards = list(shards)
        return real(X, shards, None if b2 is None else np.asarray(b2) * len(shards), R, act)
    monkeypatch.setattr(oracle, "ffn_forward_sharded", b2_per_shard)
    _expect_fail(pins.check_ffn_sharding_invariance)


def test_dropped_residual_is_caught(monkeypatch):
    real = tb.ffn_forward

    def no_residual(X, W1, b1, W2, b2, R, act="gelu"):
        return real(X, W1, b1, W2, b2, None, act)
    monkeypatch.setattr(oracle, "ffn_forward", no_residual)
    _expect_fail(pins.check_ffn_brute_force)


def test_transposed_wo_is_caught(monkeypatch):
    real = tb.attn_forward

    def wo_transposed(X, Wq, Wk, Wv, Wo, bo, R, B, S, H, d, causal=True, rows=None, bqkv=None):
        return real(X, Wq, Wk, Wv, np.asarray(Wo).T, bo, R, B, S, H, d, causal, rows, bqkv)
    monkeypatch.setattr(oracle, "attn_forward", wo_transposed)
    _expect_fail(pins.check_attention_sharding_and_heads)


def test_missing_layernorm_in_layer_is_caught(monkeypatch):
    def identity_ln(x, g, b, eps=1e-5):
        return np.asarray(x, float)
    monkeypatch.setattr(tb, "layernorm", identity_ln)
    _expect_fail(pins.check_layer)


def test_gelu_grad_without_density_term_is_caught(monkeypatch):
    # Phi(z) alone, the derivative with the z phi(z) term dropped
    monkeypatch.setattr(tb, "gelu_grad", lambda z: 0.5 * (1.0 + tb._erf(np.asarray(z, float) / math.sqrt(2.0))))
    monkeypatch.setattr(oracle, "gelu_grad", tb.gelu_grad)
    monkeypatch.setitem(tb._ACT_GRAD, "gelu", tb.gelu_grad)
    _expect_fail(pins.check_gelu_grad)
    _expect_fail(pins.check_ffn_backward_finite_differences)


def test_dw2_from_preactivation_is_caught(monkeypatch):
    real = tb.ffn_backward

    def dw2_from_z(X, W1, b1, W2, dY, act="gelu"):
        g = real(X, W1, b1, W2, dY, act)
        Z = np.asarray(X, float) @ np.asarray(W1, float) + np.asarray(b1, float)
        g["dW2"] = Z.T @ np.asarray(dY, float)
        return g
    monkeypatch.setattr(oracle, "ffn_backward", dw2_from_z)
    _expect_fail(pins.check_ffn_backward_finite_differences)


def test_input_gradient_missing_a_shard_is_caught(monkeypatch):
    real = tb.ffn_backward_sharded

    def drop_last_shard_from_dx(X, shards, dY, act="gelu"):
        shards = list(shards)
        dX, dW1, db1, dW2, db2 = real(X, shards, dY, act)
        W1_l, b1_l, W2_l = shards[-1]
        dX_l, *_ = real(X, [shards[-1]], dY, act)
        return dX - dX_l if len(shards) > 1 else dX, dW1, db1, dW2, db2
    monkeypatch.setattr(oracle, "ffn_backward_sharded", drop_last_shard_from_dx)
    _expect_fail(pins.check_ffn_backward_sharding)


def test_attention_backward_without_row_correction_is_caught(monkeypatch):
    # dS = P * dP, the softmax Jacobian's rowsum(P * dP) term dropped
    def bad(Q, K, V, dO, causal):
        Q, K, V, dO = (np.asarray(x, float) for x in (Q, K, V, dO))
        S, Hn, d = Q.shape
        scale = 1.0 / math.sqrt(d)
        keep = (np.arange(S)[None, :] <= np.arange(S)[:, None]) if causal else np.ones((S, S), bool)
        dQ, dK, dV = (np.empty_like(Q) for _ in range(3))
        for g in range(Hn):
            s = np.where(keep, (Q[:, g] @ K[:, g].T) * scale, -np.inf)
            p = np.exp(s - s.max(axis=1, keepdims=True))
            p = p / p.sum(axis=1, keepdims=True)
            dV[:, g] = p.T @ dO[:, g]
            ds = p * (dO[:, g] @ V[:, g].T)
            dQ[:, g] = ds @ K[:, g] * scale
            dK[:, g] = ds.T @ Q[:, g] * scale
        return dQ, dK, dV
    monkeypatch.setattr(tb, "attention_heads_backward", bad)
    monkeypatch.setattr(oracle, "attention_heads_backward", bad)
    _expect_fail(lambda: pins.check_attn_backward_finite_differences(True))


def test_attention_backward_transposed_dk_is_caught(monkeypatch):
    real = tb.attention_heads_backward

    def swapped(Q, K, V, dO, causal):
        dQ, dK, dV = real(Q, K, V, dO, causal)
        return dK, dQ, dV
    monkeypatch.setattr(tb, "attention_heads_backward", swapped)
    _expect_fail(lambda: pins.check_attn_backward_finite_differences(True))


def test_attention_backward_group_sum_missing_a_shard_is_caught(monkeypatch):
    real = tb.attn_backward_sharded

    def first_shard_only_dx(X, Wqkv, Wo, dY, B, S, Hg, d, causal=True, bqkv_shards=None):
        out = list(real(X, Wqkv, Wo, dY, B, S, Hg, d, causal, bqkv_shards))
        if len(Wqkv) > 1:
            out[0] = real(X, Wqkv[:1], Wo[:1], dY, B, S, Hg, d, causal,
                          None if bqkv_shards is None else bqkv_shards[:1])[0]
        return tuple(out)
    monkeypatch.setattr(oracle, "attn_backward_sharded", first_shard_only_dx)
    _expect_fail(pins.check_attn_backward_sharding)
