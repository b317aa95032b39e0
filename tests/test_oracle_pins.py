"""Pins of the fp64 oracle against what the page and the mathematics fix (CPU only).

Each check is chosen so that a plausible mistake in the oracle (tanh GeLU,
bias added per shard, 1/d instead of 1/sqrt(d), unbiased variance, a dropped
residual, a transposed operand, a wrong causal boundary) fails at least one of
them; ``test_oracle_mutations.py`` plants those mistakes to prove it.

Sources: "Tensor Parallelism > Combining Column and Row Parallelism"
(mbrenndoerfer.com) [TP-CR]; the standard normal table in
``tests/golden/normal_cdf.txt``.
"""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from megatron_tensor_transformer_bias_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _phi_table():
    rows = []
    with open(os.path.join(GOLDEN, "normal_cdf.txt")) as fh:
        for line in fh:
            line = line.strip()
            if line and not line.startswith("#"):
                x, p = line.split()
                rows.append((float(x), float(p)))
    return rows


def _np(t):
    return t.double().numpy()


# ---------------------------------------------------------------- GeLU
def check_gelu_table():
    for x, phi in _phi_table():
        assert abs(oracle.gelu(x) - x * phi) <= 1e-15 * abs(x), (x, oracle.gelu(x), x * phi)
        # Phi(-x) = 1 - Phi(x): GeLU(-x) = -x (1 - Phi(x))
        assert abs(oracle.gelu(-x) - (-x) * (1.0 - phi)) <= 2e-15 * abs(x), x


def check_gelu_identities():
    assert oracle.gelu(0.0) == 0.0
    x = np.linspace(-6, 6, 1001)
    # GeLU(x) - GeLU(-x) = x exactly, since Phi(x) + Phi(-x) = 1
    np.testing.assert_allclose(oracle.gelu(x) - oracle.gelu(-x), x, rtol=0, atol=1e-14)
    # GeLU(x) -> x for large x, -> 0 for very negative x
    assert abs(oracle.gelu(12.0) - 12.0) < 1e-15 * 12
    assert abs(oracle.gelu(-12.0)) < 1e-30


def test_gelu_table():
    check_gelu_table()


def test_gelu_identities():
    check_gelu_identities()


def test_gelu_matches_library_exact_gelu():
    z = torch.randn(4096, dtype=torch.float64, generator=torch.Generator().manual_seed(3)) * 3
    ref = F.gelu(z, approximate="none").numpy()
    np.testing.assert_allclose(oracle.gelu(z.numpy()), ref, rtol=1e-13, atol=1e-15)


def test_relu():
    z = np.array([-2.0, -0.0, 0.0, 0.5, 3.0])
    np.testing.assert_array_equal(oracle.relu(z), [0.0, 0.0, 0.0, 0.5, 3.0])


# ---------------------------------------------------------------- FFN
def _brute_ffn(X, W1, b1, W2, b2, R):
    """Pure-Python loops on tiny sizes, with math.erf."""
    M, h = len(X), len(X[0])
    f = len(W1[0])
    out = [[0.0] * h for _ in range(M)]
    for r in range(M):
        zh = []
        for j in range(f):
            z = b1[j]
            for k in range(h):
                z += X[r][k] * W1[k][j]
            zh.append(z * 0.5 * (1.0 + math.erf(z / math.sqrt(2.0))))
        for c in range(h):
            y = b2[c] + R[r][c]
            for j in range(f):
                y += zh[j] * W2[j][c]
            out[r][c] = y
    return np.array(out)


def _tiny_ffn(M=3, h=4, f=6, seed=11):
    d = inputs.ffn_inputs(M, h, f, "fp32", seed=seed)
    return {k: _np(v) for k, v in d.items()}


def _shards(W1, b1, W2, t):
    f = W1.shape[1]
    n = f // t
    return [(W1[:, i * n:(i + 1) * n], None if b1 is None else b1[i * n:(i + 1) * n],
             W2[i * n:(i + 1) * n, :]) for i in range(t)]


def check_ffn_brute_force():
    p = _tiny_ffn()
    ref = _brute_ffn(p["X"].tolist(), p["W1"].tolist(), p["b1"].tolist(), p["W2"].tolist(),
                     p["b2"].tolist(), p["X"].tolist())
    got = oracle.ffn_forward(p["X"], p["W1"], p["b1"], p["W2"], p["b2"], p["X"])
    np.testing.assert_allclose(got, ref, rtol=1e-13, atol=1e-13)
    for t in (1, 2, 3, 6):
        got_t = oracle.ffn_forward_sharded(p["X"], _shards(p["W1"], p["b1"], p["W2"], t),
                                           p["b2"], p["X"])
        np.testing.assert_allclose(got_t, ref, rtol=1e-13, atol=1e-13)


def test_ffn_brute_force_tiny():
    check_ffn_brute_force()


def check_ffn_sharding_invariance():
    # the tiny fp32 FFN workload: M=8, h=64, f=256
    p = {k: _np(v) for k, v in inputs.ffn_inputs(8, 64, 256, "fp32", seed=0).items()}
    ref = oracle.ffn_forward(p["X"], p["W1"], p["b1"], p["W2"], p["b2"], p["X"])
    for t in (1, 2, 4, 8, 16):
        got = oracle.ffn_forward_sharded(p["X"], _shards(p["W1"], p["b1"], p["W2"], t),
                                         p["b2"], p["X"])
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_ffn_sharding_invariance():
    """[TP-CR] steps 1-3 and the chaining paragraph: the sharded block equals the plain block."""
    check_ffn_sharding_invariance()


def test_ffn_special_cases():
    p = _tiny_ffn(M=4, h=8, f=16, seed=5)
    X, W1, b1, W2, b2 = p["X"], p["W1"], p["b1"], p["W2"], p["b2"]
    R = X
    # W2 = 0: out = b2 + R exactly
    out = oracle.ffn_forward_sharded(X, _shards(W1, b1, np.zeros_like(W2), 4), b2, R)
    np.testing.assert_array_equal(out, b2[None, :] + R)
    # X = 0 and b1 on table points: out = sum_j b1_j Phi(b1_j) W2[j] + b2 (+ R = 0)
    tab = _phi_table()
    b1t = np.array([x for x, _ in tab] + [-x for x, _ in tab] + [0.0] * 4)
    g = np.array([x * p_ for x, p_ in tab] + [-x * (1 - p_) for x, p_ in tab] + [0.0] * 4)
    X0 = np.zeros_like(X)
    out = oracle.ffn_forward_sharded(X0, _shards(W1, b1t, W2, 2), b2, X0)
    expect = np.tile(g @ W2 + b2, (X.shape[0], 1))
    np.testing.assert_allclose(out, expect, rtol=1e-14, atol=1e-15)
    # identity W1 and W2 (h = f): out = GeLU(X + b1) + b2 + R, element by element
    h = 8
    I = np.eye(h)
    Xt = np.array([[x for x, _ in tab] + [0.0, -1.0]] * 2)
    bz = np.zeros(h)
    out = oracle.ffn_forward(Xt, I, bz, I, bz, None)
    phi = dict(tab)
    for c, x in enumerate(Xt[0]):
        want = 0.0 if x == 0 else (x * phi[x] if x > 0 else x * (1 - phi[-x]))
        assert abs(out[0, c] - want) < 1e-15
    # doubling the shards with halved W2 gives the same block
    sh = _shards(W1, b1, W2, 2)
    doubled = [(a, b, w / 2) for (a, b, w) in sh for _ in range(2)]
    np.testing.assert_allclose(oracle.ffn_forward_sharded(X, doubled, b2, R),
                               oracle.ffn_forward_sharded(X, sh, b2, R), rtol=0, atol=1e-14)


def test_ffn_b2_added_once():
    """Reading: b2 enters once, after the sum over shards (adding it per shard gives t*b2)."""
    p = _tiny_ffn(M=2, h=4, f=8, seed=2)
    zero = np.zeros_like(p["W2"])
    for t in (1, 2, 4):
        out = oracle.ffn_forward_sharded(p["X"], _shards(p["W1"], p["b1"], zero, t), p["b2"], None)
        np.testing.assert_array_equal(out, np.tile(p["b2"], (2, 1)))


def test_reduce_partials():
    rng = np.random.default_rng(0)
    P = rng.standard_normal((3, 5, 7))
    b = rng.standard_normal(7)
    R = rng.standard_normal((5, 7))
    got = oracle.reduce_partials(list(P), b, R)
    want = np.array([[P[0, i, j] + P[1, i, j] + P[2, i, j] + b[j] + R[i, j] for j in range(7)]
                     for i in range(5)])
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-14)


# ---------------------------------------------------------------- LayerNorm
def check_layernorm():
    # hand example: x = [1,2,3,4], mean 2.5, biased variance 1.25
    x = np.array([[1.0, 2.0, 3.0, 4.0]])
    eps = 1e-5
    want = (x - 2.5) / math.sqrt(1.25 + eps)
    np.testing.assert_allclose(oracle.layernorm(x, None, None, eps), want, rtol=1e-15)
    rng = np.random.default_rng(1)
    x = rng.standard_normal((6, 64)) * 3 + 1
    y = oracle.layernorm(x, np.ones(64), np.zeros(64), eps)
    var = x.var(axis=1)
    np.testing.assert_allclose(y.mean(axis=1), 0, atol=1e-14)
    np.testing.assert_allclose((y ** 2).mean(axis=1), var / (var + eps), rtol=1e-13)
    # shift invariance LN(x + c) = LN(x)
    np.testing.assert_allclose(oracle.layernorm(x + 7.0, None, None, eps),
                               oracle.layernorm(x, None, None, eps), atol=1e-12)
    # gamma/beta are applied after normalisation
    g = rng.standard_normal(64)
    b = rng.standard_normal(64)
    np.testing.assert_allclose(oracle.layernorm(x, g, b, eps),
                               oracle.layernorm(x, None, None, eps) * g + b, rtol=1e-14, atol=1e-14)
    # a library LayerNorm (biased variance, eps inside the root)
    ref = F.layer_norm(torch.from_numpy(x), (64,), torch.from_numpy(g), torch.from_numpy(b), eps)
    np.testing.assert_allclose(oracle.layernorm(x, g, b, eps), ref.numpy(), rtol=1e-12, atol=1e-12)


def test_layernorm():
    check_layernorm()


def test_layernorm_not_shardable():
    """Negative control: LN over feature shards differs from LN over the full row."""
    rng = np.random.default_rng(2)
    x = rng.standard_normal((4, 16)) + np.linspace(-3, 3, 16)
    full = oracle.layernorm(x, None, None)
    per_shard = np.concatenate([oracle.layernorm(x[:, i * 4:(i + 1) * 4], None, None)
                                for i in range(4)], axis=1)
    assert np.abs(full - per_shard).max() > 0.1


# ---------------------------------------------------------------- attention
def _brute_attention(Q, K, V, causal):
    """Pure-Python loops: Q [nq][Hn][d], K/V [S][Hn][d]."""
    nq, Hn, d = len(Q), len(Q[0]), len(Q[0][0])
    S = len(K)
    O = np.zeros((nq, Hn, d))
    for g in range(Hn):
        for i in range(nq):
            js = [j for j in range(S) if (not causal or j <= i)]
            s = [sum(Q[i][g][k] * K[j][g][k] for k in range(d)) / math.sqrt(d) for j in js]
            m = max(s)
            e = [math.exp(v - m) for v in s]
            z = sum(e)
            for k in range(d):
                O[i, g, k] = sum(e[a] * V[js[a]][g][k] for a in range(len(js))) / z
    return O


def check_attention_core():
    rng = np.random.default_rng(4)
    for causal in (True, False):
        Q = rng.standard_normal((5, 2, 3))
        K = rng.standard_normal((5, 2, 3))
        V = rng.standard_normal((5, 2, 3))
        got = oracle.attention_heads(Q, K, V, causal)
        np.testing.assert_allclose(got, _brute_attention(Q.tolist(), K.tolist(), V.tolist(), causal),
                                   rtol=1e-13, atol=1e-13)
        # a library scaled-dot-product attention ([heads, seq, d] layout)
        ref = F.scaled_dot_product_attention(torch.from_numpy(Q).transpose(0, 1),
                                             torch.from_numpy(K).transpose(0, 1),
                                             torch.from_numpy(V).transpose(0, 1),
                                             is_causal=causal).transpose(0, 1).numpy()
        np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)
    # causal row 0 sees only key 0: O_0 = V_0
    Q = rng.standard_normal((6, 3, 4))
    K = rng.standard_normal((6, 3, 4))
    V = rng.standard_normal((6, 3, 4))
    O = oracle.attention_heads(Q, K, V, True)
    np.testing.assert_allclose(O[0], V[0], rtol=0, atol=1e-15)
    # Q = 0: uniform weights, so O_i is the mean of V over the visible prefix
    O = oracle.attention_heads(np.zeros_like(Q), K, V, True)
    prefix = np.cumsum(V, axis=0) / np.arange(1, 7)[:, None, None]
    np.testing.assert_allclose(O, prefix, rtol=1e-14, atol=1e-14)
    # V = 1: softmax rows sum to one
    O = oracle.attention_heads(Q, K, np.ones_like(V), False)
    np.testing.assert_allclose(O, 1.0, rtol=1e-14)


def test_attention_core():
    check_attention_core()


def _tiny_attn(B=2, S=6, h=16, H=4, d=4, seed=7):
    a = inputs.attn_inputs(B, S, h, H, d, seed=seed)
    return {k: _np(v) for k, v in a.items()}


def _attn_shards(a, t, H, d, perm=None):
    Hg = H // t
    n = Hg * d
    order = list(range(t)) if perm is None else perm
    Wqkv, Wo = [], []
    for i in order:
        cols = slice(i * n, (i + 1) * n)
        Wqkv.append(np.concatenate([a["Wq"][:, cols], a["Wk"][:, cols], a["Wv"][:, cols]], axis=1))
        Wo.append(a["Wo"][cols, :])
    return Wqkv, Wo


def check_attention_sharding_and_heads():
    B, S, h, H, d = 2, 6, 16, 4, 4
    a = _tiny_attn(B, S, h, H, d)
    ref = oracle.attn_forward(a["X"], a["Wq"], a["Wk"], a["Wv"], a["Wo"], a["bo"], a["X"],
                              B, S, H, d, causal=True)
    # a library reference of the whole sub-layer
    X = torch.from_numpy(a["X"]).view(B, S, h)
    q = (X @ torch.from_numpy(a["Wq"])).view(B, S, H, d).transpose(1, 2)
    k = (X @ torch.from_numpy(a["Wk"])).view(B, S, H, d).transpose(1, 2)
    v = (X @ torch.from_numpy(a["Wv"])).view(B, S, H, d).transpose(1, 2)
    o = F.scaled_dot_product_attention(q, k, v, is_causal=True).transpose(1, 2).reshape(B * S, H * d)
    lib = (o @ torch.from_numpy(a["Wo"]) + torch.from_numpy(a["bo"]) + torch.from_numpy(a["X"])).numpy()
    np.testing.assert_allclose(ref, lib, rtol=1e-12, atol=1e-12)
    for t in (1, 2, 4):
        Wqkv, Wo = _attn_shards(a, t, H, d)
        got = oracle.attn_forward_sharded(a["X"], Wqkv, Wo, a["bo"], a["X"], B, S, H // t, d, True)
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    # head independence: permuting head groups across shards (with their Wo rows)
    Wqkv, Wo = _attn_shards(a, 4, H, d, perm=[2, 0, 3, 1])
    got = oracle.attn_forward_sharded(a["X"], Wqkv, Wo, a["bo"], a["X"], B, S, 1, d, True)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    # sampled rows equal the full computation at those rows
    rows = inputs.sample_rows(B * S, 5, seq=S)
    got = oracle.attn_forward(a["X"], a["Wq"], a["Wk"], a["Wv"], a["Wo"], a["bo"], a["X"],
                              B, S, H, d, causal=True, rows=rows)
    np.testing.assert_allclose(got, ref[rows], rtol=0, atol=1e-13)
    # causal first token of each sequence: out = X_0 Wv Wo + bo + X_0
    for b in range(B):
        r = b * S
        want = a["X"][r] @ a["Wv"] @ a["Wo"] + a["bo"] + a["X"][r]
        np.testing.assert_allclose(ref[r], want, rtol=1e-13, atol=1e-13)


def test_attention_sharding_and_heads():
    check_attention_sharding_and_heads()


def test_attention_noncausal_library():
    B, S, h, H, d = 1, 5, 8, 2, 4
    a = _tiny_attn(B, S, h, H, d, seed=9)
    got = oracle.attn_forward(a["X"], a["Wq"], a["Wk"], a["Wv"], a["Wo"], None, None,
                              B, S, H, d, causal=False)
    X = torch.from_numpy(a["X"]).view(B, S, h)
    q = (X @ torch.from_numpy(a["Wq"])).view(B, S, H, d).transpose(1, 2)
    k = (X @ torch.from_numpy(a["Wk"])).view(B, S, H, d).transpose(1, 2)
    v = (X @ torch.from_numpy(a["Wv"])).view(B, S, H, d).transpose(1, 2)
    o = F.scaled_dot_product_attention(q, k, v).transpose(1, 2).reshape(B * S, H * d)
    np.testing.assert_allclose(got, (o @ torch.from_numpy(a["Wo"])).numpy(), rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- layer
def check_layer():
    B, S, h, H, d, f = 2, 5, 16, 4, 4, 32
    p = {k: _np(v) for k, v in inputs.layer_inputs(B, S, h, H, d, f, seed=3).items()}
    rng = np.random.default_rng(8)
    p["ln1_g"] = 1 + 0.1 * rng.standard_normal(h)
    p["ln1_b"] = 0.1 * rng.standard_normal(h)
    p["ln2_g"] = 1 + 0.1 * rng.standard_normal(h)
    p["ln2_b"] = 0.1 * rng.standard_normal(h)
    X = p["X"]
    got = oracle.layer_forward(X, p, B, S, H, d, eps=1e-5, causal=True)
    T = {k: torch.from_numpy(v) for k, v in p.items()}
    x = T["X"]
    a = F.layer_norm(x, (h,), T["ln1_g"], T["ln1_b"], 1e-5).view(B, S, h)
    q = (a @ T["Wq"]).view(B, S, H, d).transpose(1, 2)
    k = (a @ T["Wk"]).view(B, S, H, d).transpose(1, 2)
    v = (a @ T["Wv"]).view(B, S, H, d).transpose(1, 2)
    o = F.scaled_dot_product_attention(q, k, v, is_causal=True).transpose(1, 2).reshape(B * S, H * d)
    h1 = x + o @ T["Wo"] + T["bo"]
    a2 = F.layer_norm(h1, (h,), T["ln2_g"], T["ln2_b"], 1e-5)
    lib = h1 + F.gelu(a2 @ T["W1"] + T["b1"]) @ T["W2"] + T["b2"]
    np.testing.assert_allclose(got, lib.numpy(), rtol=1e-12, atol=1e-12)
    rows = inputs.sample_rows(B * S, 4, seq=S)
    np.testing.assert_allclose(oracle.layer_forward(X, p, B, S, H, d, rows=rows), got[rows],
                               rtol=0, atol=1e-13)
    # zero projections: out = X + bo + b2
    z = dict(p)
    z["Wo"] = np.zeros_like(p["Wo"])
    z["W2"] = np.zeros_like(p["W2"])
    np.testing.assert_allclose(oracle.layer_forward(X, z, B, S, H, d), X + p["bo"] + p["b2"],
                               rtol=0, atol=1e-15)


def test_layer():
    check_layer()


def test_sample_rows():
    rows = inputs.sample_rows(4096, 64, seq=2048)
    assert len(rows) == 64 and len(set(rows)) == 64
    assert {0, 2047, 2048, 4095} <= set(rows)
    assert rows == inputs.sample_rows(4096, 64, seq=2048)
    assert inputs.sample_rows(5, 64) == [0, 1, 2, 3, 4]


# ---------------------------------------------------------------- FFN backward
def _normal_density(x):
    return math.exp(-0.5 * x * x) / math.sqrt(2.0 * math.pi)


def check_gelu_grad():
    """GeLU'(x) = Phi(x) + x phi(x): Phi from the printed normal table (not from erf),
    phi the normal density; GeLU'(0) = 1/2; GeLU'(x) + GeLU'(-x) = 1 (derivative of
    GeLU(x) - GeLU(-x) = x); -> 1 and -> 0 in the tails; and the derivative of the
    oracle's own GeLU by central differences."""
    for x, phi in _phi_table():
        want = phi + x * _normal_density(x)
        assert abs(oracle.gelu_grad(x) - want) <= 1e-14, (x, oracle.gelu_grad(x), want)
        want_neg = (1.0 - phi) - x * _normal_density(x)
        assert abs(oracle.gelu_grad(-x) - want_neg) <= 1e-14, x
    assert oracle.gelu_grad(0.0) == 0.5
    x = np.linspace(-7, 7, 1401)
    np.testing.assert_allclose(oracle.gelu_grad(x) + oracle.gelu_grad(-x), 1.0, rtol=0, atol=1e-14)
    assert abs(oracle.gelu_grad(12.0) - 1.0) < 1e-15 and abs(oracle.gelu_grad(-12.0)) < 1e-15
    h = 1e-5
    fd = (oracle.gelu(x + h) - oracle.gelu(x - h)) / (2 * h)
    np.testing.assert_allclose(oracle.gelu_grad(x), fd, rtol=0, atol=1e-9)


def test_gelu_grad():
    check_gelu_grad()


def test_relu_grad():
    np.testing.assert_array_equal(oracle.relu_grad(np.array([-1.0, 0.0, 1e-30, 2.0])), [0.0, 0.0, 1.0, 1.0])


def _tiny_backward_case(seed=21, M=3, h=4, f=6):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((M, h)), rng.standard_normal((h, f)) * 0.5, rng.standard_normal(f) * 0.3,
            rng.standard_normal((f, h)) * 0.5, rng.standard_normal(h) * 0.3, rng.standard_normal((M, h)))


def check_ffn_backward_finite_differences(act="gelu"):
    """Every gradient entry of L = sum(dY * out) against a central difference of the
    oracle's own forward, on a tiny block (no shared code with the backward)."""
    X, W1, b1, W2, b2, dY = _tiny_backward_case()
    g = oracle.ffn_backward(X, W1, b1, W2, dY, act=act)

    def loss(X_, W1_, b1_, W2_, b2_):
        return float(np.sum(dY * oracle.ffn_forward(X_, W1_, b1_, W2_, b2_, None, act=act)))

    args = [X, W1, b1, W2, b2]
    names = ["dX", "dW1", "db1", "dW2", "db2"]
    eps = 1e-6
    for k, name in enumerate(names):
        a = args[k]
        fd = np.zeros_like(a)
        for idx in np.ndindex(a.shape):
            up = [x.copy() for x in args]
            dn = [x.copy() for x in args]
            up[k][idx] += eps
            dn[k][idx] -= eps
            fd[idx] = (loss(*up) - loss(*dn)) / (2 * eps)
        np.testing.assert_allclose(g[name], fd, rtol=1e-6, atol=1e-7, err_msg=name)


def test_ffn_backward_finite_differences():
    check_ffn_backward_finite_differences("gelu")
    check_ffn_backward_finite_differences("relu")


def test_ffn_backward_matches_float64_autograd():
    X, W1, b1, W2, b2, dY = _tiny_backward_case(seed=22, M=5, h=8, f=12)
    t = [torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (X, W1, b1, W2, b2)]
    out = F.gelu(t[0] @ t[1] + t[2], approximate="none") @ t[3] + t[4]
    out.backward(torch.tensor(dY))
    g = oracle.ffn_backward(X, W1, b1, W2, dY)
    for name, tt in zip(["dX", "dW1", "db1", "dW2", "db2"], t):
        np.testing.assert_allclose(g[name], tt.grad.numpy(), rtol=1e-12, atol=1e-13, err_msg=name)


def check_ffn_backward_sharding():
    """The shard-by-shard backward (local row-layer gradients, one ordered sum for the
    input gradient) equals the unsharded chain rule for every t dividing f."""
    X, W1, b1, W2, b2, dY = _tiny_backward_case(seed=23, M=7, h=8, f=24)
    g = oracle.ffn_backward(X, W1, b1, W2, dY)
    for t in (1, 2, 3, 4, 6, 8, 12, 24):
        n = 24 // t
        shards = [(W1[:, i * n:(i + 1) * n], b1[i * n:(i + 1) * n], W2[i * n:(i + 1) * n]) for i in range(t)]
        dX, dW1, db1, dW2, db2 = oracle.ffn_backward_sharded(X, shards, dY)
        np.testing.assert_allclose(dX, g["dX"], rtol=0, atol=1e-12)
        np.testing.assert_allclose(np.concatenate(dW1, axis=1), g["dW1"], rtol=0, atol=1e-12)
        np.testing.assert_allclose(np.concatenate(db1), g["db1"], rtol=0, atol=1e-12)
        np.testing.assert_allclose(np.concatenate(dW2, axis=0), g["dW2"], rtol=0, atol=1e-12)
        np.testing.assert_allclose(db2, g["db2"], rtol=0, atol=1e-12)


def test_ffn_backward_sharding():
    check_ffn_backward_sharding()


def test_ffn_backward_special_cases():
    X, W1, b1, W2, b2, dY = _tiny_backward_case(seed=24)
    z = oracle.ffn_backward(X, W1, b1, W2, np.zeros_like(dY))
    for v in z.values():
        assert not np.any(v)
    # W2 = 0: nothing flows back into the column layer; the row layer still gets A^T dY
    g = oracle.ffn_backward(X, W1, b1, np.zeros_like(W2), dY)
    assert not np.any(g["dX"]) and not np.any(g["dW1"]) and not np.any(g["db1"])
    A = oracle.gelu(X @ W1 + b1)
    np.testing.assert_allclose(g["dW2"], A.T @ dY, rtol=1e-14)
    np.testing.assert_allclose(g["db2"], dY.sum(0), rtol=1e-14)


# ------------------------------------------------------------------ attention backward
def _tiny_attn_backward_case(seed=31, B=2, S=5, h=8, H=2, d=4):
    rng = np.random.default_rng(seed)
    return {"X": rng.standard_normal((B * S, h)), "Wq": rng.standard_normal((h, H * d)) * 0.5,
            "Wk": rng.standard_normal((h, H * d)) * 0.5, "Wv": rng.standard_normal((h, H * d)) * 0.5,
            "Wo": rng.standard_normal((H * d, h)) * 0.5, "bo": rng.standard_normal(h) * 0.3,
            "bq": rng.standard_normal(H * d) * 0.3, "bk": rng.standard_normal(H * d) * 0.3,
            "bv": rng.standard_normal(H * d) * 0.3, "dY": rng.standard_normal((B * S, h))}


def check_attn_backward_finite_differences(causal=True):
    """Every gradient entry of L = sum(dY * out) against a central difference of the
    forward oracle (attn_forward), which shares no code with the backward."""
    B, S, h, H, d = 2, 5, 8, 2, 4
    a = _tiny_attn_backward_case(B=B, S=S, h=h, H=H, d=d)
    g = oracle.attn_backward(a["X"], a["Wq"], a["Wk"], a["Wv"], a["Wo"], a["dY"], B, S, H, d, causal,
                             bqkv=(a["bq"], a["bk"], a["bv"]))
    names = ["X", "Wq", "Wk", "Wv", "Wo", "bo", "bq", "bk", "bv"]

    def loss(p):
        out = oracle.attn_forward(p["X"], p["Wq"], p["Wk"], p["Wv"], p["Wo"], p["bo"], None, B, S, H, d,
                                  causal, bqkv=(p["bq"], p["bk"], p["bv"]))
        return float(np.sum(a["dY"] * out))

    eps = 1e-6
    for name in names:
        fd = np.zeros_like(a[name])
        for idx in np.ndindex(a[name].shape):
            up = dict(a); dn = dict(a)
            up[name] = a[name].copy(); dn[name] = a[name].copy()
            up[name][idx] += eps
            dn[name][idx] -= eps
            fd[idx] = (loss(up) - loss(dn)) / (2 * eps)
        np.testing.assert_allclose(g["d" + name], fd, rtol=1e-6, atol=1e-7, err_msg=name)


def test_attn_backward_finite_differences():
    check_attn_backward_finite_differences(True)
    check_attn_backward_finite_differences(False)


def test_attn_backward_matches_float64_autograd():
    """Against autograd through torch's own scaled_dot_product_attention in float64."""
    B, S, h, H, d = 2, 7, 16, 4, 4
    a = _tiny_attn_backward_case(seed=32, B=B, S=S, h=h, H=H, d=d)
    for causal in (True, False):
        t = {k: torch.tensor(a[k], dtype=torch.float64, requires_grad=True)
             for k in ("X", "Wq", "Wk", "Wv", "Wo", "bo", "bq", "bk", "bv")}
        X = t["X"].view(B, S, h)
        q = (X @ t["Wq"] + t["bq"]).view(B, S, H, d).transpose(1, 2)
        k = (X @ t["Wk"] + t["bk"]).view(B, S, H, d).transpose(1, 2)
        v = (X @ t["Wv"] + t["bv"]).view(B, S, H, d).transpose(1, 2)
        o = F.scaled_dot_product_attention(q, k, v, is_causal=causal).transpose(1, 2).reshape(B * S, H * d)
        out = o @ t["Wo"] + t["bo"]
        out.backward(torch.tensor(a["dY"]))
        g = oracle.attn_backward(a["X"], a["Wq"], a["Wk"], a["Wv"], a["Wo"], a["dY"], B, S, H, d, causal,
                                 bqkv=(a["bq"], a["bk"], a["bv"]))
        for name in t:
            np.testing.assert_allclose(g["d" + name], t[name].grad.numpy(), rtol=1e-11, atol=1e-12,
                                       err_msg=f"{name} causal={causal}")


def check_attn_backward_sharding():
    """Head group by head group (local projection gradients, one ordered sum for dX) equals
    the unsharded chain rule for every t dividing H, and permuting the groups across shards
    (with their Wo rows) permutes the per-shard gradients and leaves dX, dbo unchanged."""
    B, S, h, H, d = 2, 6, 16, 4, 4
    a = _tiny_attn_backward_case(seed=33, B=B, S=S, h=h, H=H, d=d)
    g = oracle.attn_backward(a["X"], a["Wq"], a["Wk"], a["Wv"], a["Wo"], a["dY"], B, S, H, d, True,
                             bqkv=(a["bq"], a["bk"], a["bv"]))
    for t, perm in ((1, None), (2, None), (4, None), (4, [2, 0, 3, 1])):
        n = (H // t) * d
        order = list(range(t)) if perm is None else perm
        Wqkv, Wo, bqkv = [], [], []
        for i in order:
            cols = slice(i * n, (i + 1) * n)
            Wqkv.append(np.concatenate([a["Wq"][:, cols], a["Wk"][:, cols], a["Wv"][:, cols]], axis=1))
            bqkv.append(np.concatenate([a["bq"][cols], a["bk"][cols], a["bv"][cols]]))
            Wo.append(a["Wo"][cols, :])
        dX, dWqkv, dbqkv, dWo, dbo = oracle.attn_backward_sharded(a["X"], Wqkv, Wo, a["dY"], B, S, H // t, d,
                                                                  True, bqkv_shards=bqkv)
        np.testing.assert_allclose(dX, g["dX"], rtol=0, atol=1e-12)
        np.testing.assert_allclose(dbo, g["dbo"], rtol=0, atol=1e-12)
        for j, i in enumerate(order):
            cols = slice(i * n, (i + 1) * n)
            want = np.concatenate([g["dWq"][:, cols], g["dWk"][:, cols], g["dWv"][:, cols]], axis=1)
            np.testing.assert_allclose(dWqkv[j], want, rtol=0, atol=1e-12)
            want_b = np.concatenate([g["dbq"][cols], g["dbk"][cols], g["dbv"][cols]])
            np.testing.assert_allclose(dbqkv[j], want_b, rtol=0, atol=1e-12)
            np.testing.assert_allclose(dWo[j], g["dWo"][cols, :], rtol=0, atol=1e-12)


def test_attn_backward_sharding():
    check_attn_backward_sharding()


def test_attn_backward_special_cases():
    a = _tiny_attn_backward_case(seed=34)
    rng = np.random.default_rng(35)
    # one-token sequences: softmax over a single key is 1, so no gradient reaches Q or K,
    # and dV = dO
    S, Hn, d = 1, 3, 4
    Q, K, V, dO = (rng.standard_normal((S, Hn, d)) for _ in range(4))
    dQ, dK, dV = oracle.attention_heads_backward(Q, K, V, dO, True)
    assert not np.any(dQ) and not np.any(dK)
    np.testing.assert_allclose(dV, dO, rtol=0, atol=0)
    # V constant across keys: O does not depend on the scores, so dQ = dK = 0 and dV is the
    # column sums of P weighted by dO (each row of P sums to 1: sum over keys of dV = sum of dO)
    S = 6
    Q, K, dO = (rng.standard_normal((S, Hn, d)) for _ in range(3))
    V = np.broadcast_to(rng.standard_normal((1, Hn, d)), (S, Hn, d)).copy()
    for causal in (True, False):
        dQ, dK, dV = oracle.attention_heads_backward(Q, K, V, dO, causal)
        np.testing.assert_allclose(dQ, 0, atol=1e-14)
        np.testing.assert_allclose(dK, 0, atol=1e-14)
        np.testing.assert_allclose(dV.sum(axis=0), dO.sum(axis=0), rtol=1e-13, atol=1e-13)
    # causal: the last key is seen by the last query only, so its dK / dV come from that row
    dQ, dK, dV = oracle.attention_heads_backward(Q, K, rng.standard_normal((S, Hn, d)), dO, True)
    assert np.all(np.isfinite(dK))
    # dY = 0: every gradient is zero
    z = oracle.attn_backward(a["X"], a["Wq"], a["Wk"], a["Wv"], a["Wo"], np.zeros_like(a["dY"]), 2, 5, 2, 4)
    for v in z.values():
        assert not np.any(v)
