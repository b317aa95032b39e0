"""fp64 definitions of the column->row tensor-parallel block (test infrastructure only).

[TP-CR] = "Tensor Parallelism > Combining Column and Row Parallelism"
(mbrenndoerfer.com).  Readings of what the page leaves open are stated where
they are used: exact-erf GeLU; b1 split with W1's columns and b2 added once
after the sum; contiguous equal shards; shard sums taken in order 0..t-1;
softmax scale 1/sqrt(d); causal mask j <= i inside each sequence; LayerNorm
with biased variance and eps inside the square root; QKV shard layout
[Q heads | K heads | V heads] of the head group.
"""
from __future__ import annotations

import math
from typing import Iterable, Optional, Sequence, Tuple

import numpy as np
from scipy.special import erf as _erf

F64 = np.float64


def _f64(a):
    return None if a is None else np.asarray(a, dtype=F64)


# --------------------------------------------------------------------------
# Nonlinearity ([TP-CR], step 1 and the paragraph on where the nonlinearity
# fits: GeLU is applied element-wise to each shard, no communication).
# --------------------------------------------------------------------------
def gelu(z):
    """Exact GeLU, z * Phi(z) with Phi the standard normal CDF, Phi(z) = (1 + erf(z/sqrt 2)) / 2."""
    z = _f64(z)
    return z * 0.5 * (1.0 + _erf(z / math.sqrt(2.0)))


def relu(z):
    """ReLU, the alternative nonlinearity the same paragraph allows."""
    z = _f64(z)
    return np.maximum(z, 0.0)


_ACT = {"gelu": gelu, "relu": relu}


# --------------------------------------------------------------------------
# FFN block ([TP-CR] steps 1-3).
# --------------------------------------------------------------------------
def ffn_forward(X, W1, b1, W2, b2, R, act="gelu"):
    """Unsharded FFN block: out = act(X W1 + b1) W2 + b2 + R.

    Column/row chaining is exact algebra (the concatenated column shards of W1
    and the stacked row shards of W2 give back W1 and W2), so the sharded block
    reaches this result up to rounding.  b1, b2, R may be None (treated as 0).
    """
    X, W1, W2 = _f64(X), _f64(W1), _f64(W2)
    Z = X @ W1
    if b1 is not None:
        Z = Z + _f64(b1)
    Zh = _ACT[act](Z)
    Y = Zh @ W2
    if b2 is not None:
        Y = Y + _f64(b2)
    if R is not None:
        Y = Y + _f64(R)
    return Y


def ffn_forward_sharded(X, shards: Iterable[Tuple], b2, R, act="gelu"):
    """The block as the page computes it, shard by shard.

    For each shard i (taken in order 0..t-1), with ``shards`` yielding
    ``(W1_i [h, f/t], b1_i [f/t] or None, W2_i [f/t, h])``:

    * step 1: Z_i = X W1_i (+ b1_i), Zh_i = act(Z_i)  -- local, no communication;
    * step 2: Y_i = Zh_i W2_i  -- a partial sum over the full output;
    * step 3: Y = sum_i Y_i, then + b2 once and + R.
    """
    X = _f64(X)
    Y = None
    for W1_i, b1_i, W2_i in shards:
        Z_i = X @ _f64(W1_i)
        if b1_i is not None:
            Z_i = Z_i + _f64(b1_i)
        Y_i = _ACT[act](Z_i) @ _f64(W2_i)
        Y = Y_i if Y is None else Y + Y_i
    if b2 is not None:
        Y = Y + _f64(b2)
    if R is not None:
        Y = Y + _f64(R)
    return Y


def reduce_partials(P: Sequence, bias, R):
    """Step 3 on its own: sum the partials P_0..P_{t-1} in order, then + bias + R."""
    Y = None
    for p in P:
        Y = _f64(p) if Y is None else Y + _f64(p)
    if bias is not None:
        Y = Y + _f64(bias)
    if R is not None:
        Y = Y + _f64(R)
    return Y


# --------------------------------------------------------------------------
# LayerNorm: a reduction over the full feature vector (the paragraph on
# softmax and layer normalization: it needs the mean and variance over all
# features, so it runs replicated on the full row, never on a shard).
# --------------------------------------------------------------------------
def layernorm(x, g, b, eps=1e-5):
    """Per row: (x - mean) / sqrt(var + eps) * g + b, var the biased (1/h) variance."""
    x = _f64(x)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    y = (x - mu) / np.sqrt(var + eps)
    if g is not None:
        y = y * _f64(g)
    if b is not None:
        y = y + _f64(b)
    return y


# --------------------------------------------------------------------------
# Attention ([TP-CR], paragraphs on multi-head attention, head independence
# and the column split of the QKV weights).
# --------------------------------------------------------------------------
def attention_heads(Q, K, V, causal, q_pos=None):
    """Per-head scaled dot-product attention for one sequence.

    Q [nq, Hn, d], K and V [S, Hn, d]; ``q_pos`` [nq] gives each query's
    position in the sequence (default 0..nq-1).  For each head:
    scores = Q K^T / sqrt(d); with ``causal`` key j is kept only when
    j <= q_pos; P = softmax over keys, computed as exp(s - max) / sum;
    O = P V.  Returns O [nq, Hn, d].
    """
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    nq, Hn, d = Q.shape
    S = K.shape[0]
    if q_pos is None:
        q_pos = np.arange(nq)
    q_pos = np.asarray(q_pos)
    O = np.empty((nq, Hn, d), dtype=F64)
    scale = 1.0 / math.sqrt(d)
    keep = (np.arange(S)[None, :] <= q_pos[:, None]) if causal else np.ones((nq, S), bool)
    for g in range(Hn):
        s = (Q[:, g, :] @ K[:, g, :].T) * scale
        s = np.where(keep, s, -np.inf)
        m = s.max(axis=1, keepdims=True)
        p = np.exp(s - m)
        p = p / p.sum(axis=1, keepdims=True)
        O[:, g, :] = p @ V[:, g, :]
    return O


def _rows_by_sequence(rows, B, S):
    rows = np.asarray(rows)
    return [(b, rows[(rows >= b * S) & (rows < (b + 1) * S)]) for b in range(B)]


def attn_forward(X, Wq, Wk, Wv, Wo, bo, R, B, S, H, d, causal=True, rows=None, bqkv=None):
    """Unsharded attention sub-layer: out = concat_h(softmax(Q_h K_h^T/sqrt d) V_h) Wo + bo + R.

    X [B*S, h] (row r = b*S + s), Wq/Wk/Wv [h, H*d] with head g at columns
    g*d..g*d+d, Wo [H*d, h].  ``bqkv`` (optional) is (bq, bk, bv), each [H*d].
    With ``rows`` given, only those output rows are computed (their
    sequences' K and V are still formed for every token).
    """
    X = _f64(X)
    Wq, Wk, Wv, Wo = _f64(Wq), _f64(Wk), _f64(Wv), _f64(Wo)
    M = B * S
    if rows is None:
        rows = np.arange(M)
    rows = np.asarray(rows)
    O = np.empty((len(rows), H * d), dtype=F64)
    pos_in_out = {int(r): i for i, r in enumerate(rows)}
    for b, rb in _rows_by_sequence(rows, B, S):
        if len(rb) == 0:
            continue
        Xs = X[b * S:(b + 1) * S]
        Xq = X[rb]
        Q = Xq @ Wq
        K = Xs @ Wk
        V = Xs @ Wv
        if bqkv is not None:
            Q, K, V = Q + _f64(bqkv[0]), K + _f64(bqkv[1]), V + _f64(bqkv[2])
        Ob = attention_heads(Q.reshape(len(rb), H, d), K.reshape(S, H, d), V.reshape(S, H, d),
                             causal, q_pos=rb - b * S)
        for j, r in enumerate(rb):
            O[pos_in_out[int(r)]] = Ob[j].reshape(H * d)
    Y = O @ Wo
    if bo is not None:
        Y = Y + _f64(bo)
    if R is not None:
        Y = Y + _f64(R)[rows]
    return Y


def attn_forward_sharded(X, Wqkv_shards, Wo_shards, bo, R, B, S, Hg, d, causal=True):
    """The attention sub-layer as the page shards it, head group by head group.

    Shard i holds Wqkv_i [h, 3*Hg*d] = [Q heads | K heads | V heads] of its
    group (column-parallel) and Wo_i [Hg*d, h] (the matching rows of the
    output projection, row-parallel).  Each shard attends over its own heads
    only and yields a partial Y_i = O_i Wo_i; the partials are summed in
    order, then + bo once and + R.
    """
    X = _f64(X)
    Y = None
    for Wqkv_i, Wo_i in zip(Wqkv_shards, Wo_shards):
        Wqkv_i = _f64(Wqkv_i)
        n = Hg * d
        O_i = np.empty((B * S, n), dtype=F64)
        for b in range(B):
            Xs = X[b * S:(b + 1) * S]
            QKV = Xs @ Wqkv_i
            Q = QKV[:, 0:n].reshape(S, Hg, d)
            K = QKV[:, n:2 * n].reshape(S, Hg, d)
            V = QKV[:, 2 * n:3 * n].reshape(S, Hg, d)
            O_i[b * S:(b + 1) * S] = attention_heads(Q, K, V, causal).reshape(S, n)
        Y_i = O_i @ _f64(Wo_i)
        Y = Y_i if Y is None else Y + Y_i
    if bo is not None:
        Y = Y + _f64(bo)
    if R is not None:
        Y = Y + _f64(R)
    return Y


# --------------------------------------------------------------------------
# Pre-LN layer ([TP-CR], the paragraph on the two reductions per layer:
# residual connections are added to the reduced results between the
# sub-layers; the LayerNorm placement (pre-LN) is the stated layer form).
# --------------------------------------------------------------------------
def layer_forward(X, p, B, S, H, d, eps=1e-5, causal=True, rows=None):
    """h1 = X + Attn(LN1(X)); out = h1 + FFN(LN2(h1)).

    ``p`` holds Wq, Wk, Wv, Wo, bo, W1, b1, W2, b2, ln1_g, ln1_b, ln2_g, ln2_b.
    With ``rows``, only those output rows are computed; LN1 is still taken for
    every token of their sequences because attention reads them all.
    """
    X = _f64(X)
    M = B * S
    if rows is None:
        rows = np.arange(M)
    rows = np.asarray(rows)
    seqs = sorted({int(r) // S for r in rows})
    A = np.zeros_like(X) if len(seqs) == B else np.full_like(X, np.nan)
    for b in seqs:
        A[b * S:(b + 1) * S] = layernorm(X[b * S:(b + 1) * S], p["ln1_g"], p["ln1_b"], eps)
    attn_rows = attn_forward(A, p["Wq"], p["Wk"], p["Wv"], p["Wo"], p["bo"], None,
                             B, S, H, d, causal, rows=rows)
    h1 = X[rows] + attn_rows
    a2 = layernorm(h1, p["ln2_g"], p["ln2_b"], eps)
    return ffn_forward(a2, p["W1"], p["b1"], p["W2"], p["b2"], h1)


# --------------------------------------------------------------------------
# Backward pass of the FFN block.  The page describes the forward pass (one
# all-reduce per two-layer block) and notes its effect on training; the
# gradients are the chain rule taken back through steps 3, 2 and 1.  Read with
# the chaining paragraph's column/row duality: the upstream gradient dY is the
# same on every shard (it is the gradient of the forward all-reduce's output),
# so the row-parallel layer's input gradient dA_i = dY W2_i^T is local to shard
# i, while the column-parallel layer's input gradient dX = sum_i dZ_i W1_i^T is
# a sum over shards -- the backward pass's one reduction.
# --------------------------------------------------------------------------
def gelu_grad(z):
    """d/dz GeLU(z) = Phi(z) + z phi(z), phi(z) = exp(-z^2/2) / sqrt(2 pi) the normal density."""
    z = _f64(z)
    return 0.5 * (1.0 + _erf(z / math.sqrt(2.0))) + z * np.exp(-0.5 * z * z) / math.sqrt(2.0 * math.pi)


def relu_grad(z):
    """d/dz ReLU(z): 1 where z > 0, else 0 (0 at z = 0)."""
    return (_f64(z) > 0.0).astype(F64)


_ACT_GRAD = {"gelu": gelu_grad, "relu": relu_grad}


def ffn_backward(X, W1, b1, W2, dY, act="gelu"):
    """Gradients of out = act(X W1 + b1) W2 + b2 + R given dY = dL/d(out).

    Returns a dict with dX (the gradient through the FFN path only: when the
    residual R is X, the caller's total input gradient is dX + dY), dW1, db1,
    dW2 and db2:
        Z = X W1 + b1,   A = act(Z)
        dW2 = A^T dY,    db2 = sum over rows of dY
        dA = dY W2^T,    dZ = dA * act'(Z)
        dW1 = X^T dZ,    db1 = sum over rows of dZ,   dX = dZ W1^T
    """
    X, W1, W2, dY = _f64(X), _f64(W1), _f64(W2), _f64(dY)
    Z = X @ W1
    if b1 is not None:
        Z = Z + _f64(b1)
    A = _ACT[act](Z)
    dA = dY @ W2.T
    dZ = dA * _ACT_GRAD[act](Z)
    return {"dX": dZ @ W1.T, "dW1": X.T @ dZ, "db1": dZ.sum(axis=0), "dW2": A.T @ dY, "db2": dY.sum(axis=0)}


def ffn_backward_sharded(X, shards: Iterable[Tuple], dY, act="gelu"):
    """The backward pass shard by shard, for ``shards`` yielding (W1_i, b1_i or None, W2_i)
    in the order 0..t-1:

    * recompute Z_i = X W1_i (+ b1_i) and A_i = act(Z_i) (step 1 again, local);
    * dW2_i = A_i^T dY and dA_i = dY W2_i^T (the row layer's gradients, local);
    * dZ_i = dA_i * act'(Z_i), dW1_i = X^T dZ_i, db1_i = column sums of dZ_i (local);
    * dX = sum_i dZ_i W1_i^T, taken in the order 0..t-1 (the reduction);
    * db2 = column sums of dY, once.

    Returns (dX, [dW1_i], [db1_i], [dW2_i], db2)."""
    X, dY = _f64(X), _f64(dY)
    dX = None
    dW1, db1, dW2 = [], [], []
    for W1_i, b1_i, W2_i in shards:
        W1_i, W2_i = _f64(W1_i), _f64(W2_i)
        Z_i = X @ W1_i
        if b1_i is not None:
            Z_i = Z_i + _f64(b1_i)
        A_i = _ACT[act](Z_i)
        dW2.append(A_i.T @ dY)
        dZ_i = (dY @ W2_i.T) * _ACT_GRAD[act](Z_i)
        dW1.append(X.T @ dZ_i)
        db1.append(dZ_i.sum(axis=0))
        part = dZ_i @ W1_i.T
        dX = part if dX is None else dX + part
    return dX, dW1, db1, dW2, dY.sum(axis=0)


# --------------------------------------------------------------------------
# Backward pass of the attention sub-layer.  Same reading as the FFN block's:
# the chain rule back through the output projection (row-parallel: its input
# gradient dO_i = dY Wo_i^T is local to head group i), per-head attention
# (heads are independent) and the QKV projection (column-parallel: the input
# gradient dX = sum_i dQKV_i Wqkv_i^T is the one reduction over groups).
# --------------------------------------------------------------------------
def attention_heads_backward(Q, K, V, dO, causal):
    """Gradients of O = softmax(Q K^T / sqrt(d), masked) V for one sequence, head by head.

    Q, K, V, dO [S, Hn, d].  For each head, with s = Q K^T / sqrt(d) (masked
    scores -inf) and P = softmax over keys:
        dV = P^T dO,   dP = dO V^T,
        dS = P * (dP - rowsum(P * dP))      (the softmax Jacobian applied row by row),
        dQ = dS K / sqrt(d),   dK = dS^T Q / sqrt(d).
    Returns dQ, dK, dV [S, Hn, d].
    """
    Q, K, V, dO = _f64(Q), _f64(K), _f64(V), _f64(dO)
    S, Hn, d = Q.shape
    scale = 1.0 / math.sqrt(d)
    keep = (np.arange(S)[None, :] <= np.arange(S)[:, None]) if causal else np.ones((S, S), bool)
    dQ, dK, dV = (np.empty_like(Q) for _ in range(3))
    for g in range(Hn):
        s = np.where(keep, (Q[:, g, :] @ K[:, g, :].T) * scale, -np.inf)
        p = np.exp(s - s.max(axis=1, keepdims=True))
        p = p / p.sum(axis=1, keepdims=True)
        dV[:, g, :] = p.T @ dO[:, g, :]
        dp = dO[:, g, :] @ V[:, g, :].T
        ds = p * (dp - np.sum(p * dp, axis=1, keepdims=True))
        dQ[:, g, :] = ds @ K[:, g, :] * scale
        dK[:, g, :] = ds.T @ Q[:, g, :] * scale
    return dQ, dK, dV


def attn_backward(X, Wq, Wk, Wv, Wo, dY, B, S, H, d, causal=True, bqkv=None):
    """Gradients of out = concat_h(attention_h) Wo + bo + R given dY = dL/d(out).

    Returns a dict with dX (through the attention path only; with R = X the
    caller's total input gradient is dX + dY), dWq, dWk, dWv, dbq, dbk, dbv,
    dWo and dbo:
        Q = X Wq (+ bq), K = X Wk (+ bk), V = X Wv (+ bv),  O = attention(Q, K, V)
        dWo = O^T dY,   dbo = sum over rows of dY,   dO = dY Wo^T
        dQ, dK, dV = attention_heads_backward(Q, K, V, dO) per sequence
        dWq = X^T dQ (likewise K, V),  dbq = sum over rows of dQ (likewise K, V)
        dX = dQ Wq^T + dK Wk^T + dV Wv^T
    """
    X, Wq, Wk, Wv, Wo, dY = _f64(X), _f64(Wq), _f64(Wk), _f64(Wv), _f64(Wo), _f64(dY)
    M = B * S
    Q, K, V = X @ Wq, X @ Wk, X @ Wv
    if bqkv is not None:
        Q, K, V = Q + _f64(bqkv[0]), K + _f64(bqkv[1]), V + _f64(bqkv[2])
    O = np.empty((M, H * d), dtype=F64)
    for b in range(B):
        sl = slice(b * S, (b + 1) * S)
        O[sl] = attention_heads(Q[sl].reshape(S, H, d), K[sl].reshape(S, H, d), V[sl].reshape(S, H, d),
                                causal).reshape(S, H * d)
    dO = dY @ Wo.T
    dQ, dK, dV = (np.empty((M, H * d), dtype=F64) for _ in range(3))
    for b in range(B):
        sl = slice(b * S, (b + 1) * S)
        gq, gk, gv = attention_heads_backward(Q[sl].reshape(S, H, d), K[sl].reshape(S, H, d),
                                              V[sl].reshape(S, H, d), dO[sl].reshape(S, H, d), causal)
        dQ[sl], dK[sl], dV[sl] = gq.reshape(S, H * d), gk.reshape(S, H * d), gv.reshape(S, H * d)
    return {"dX": dQ @ Wq.T + dK @ Wk.T + dV @ Wv.T,
            "dWq": X.T @ dQ, "dWk": X.T @ dK, "dWv": X.T @ dV,
            "dbq": dQ.sum(axis=0), "dbk": dK.sum(axis=0), "dbv": dV.sum(axis=0),
            "dWo": O.T @ dY, "dbo": dY.sum(axis=0)}


def attn_backward_sharded(X, Wqkv_shards, Wo_shards, dY, B, S, Hg, d, causal=True, bqkv_shards=None):
    """The backward pass head group by head group, for shards i = 0..t-1 holding
    Wqkv_i [h, 3*Hg*d] = [Q heads | K heads | V heads] (optional bias bqkv_i) and Wo_i [Hg*d, h]:

    * recompute QKV_i = X Wqkv_i (+ bqkv_i) and the group's attention output O_i (local);
    * dWo_i = O_i^T dY and dO_i = dY Wo_i^T (the row-parallel projection's gradients, local);
    * dQKV_i = [dQ | dK | dV] of the group's heads (local; heads are independent);
    * dWqkv_i = X^T dQKV_i, dbqkv_i = column sums of dQKV_i (local);
    * dX = sum_i dQKV_i Wqkv_i^T, in the order 0..t-1 (the reduction);
    * dbo = column sums of dY, once.

    Returns (dX, [dWqkv_i], [dbqkv_i], [dWo_i], dbo)."""
    X, dY = _f64(X), _f64(dY)
    M, n = B * S, Hg * d
    dX = None
    dWqkv, dbqkv, dWo = [], [], []
    for i, (Wqkv_i, Wo_i) in enumerate(zip(Wqkv_shards, Wo_shards)):
        Wqkv_i, Wo_i = _f64(Wqkv_i), _f64(Wo_i)
        QKV = X @ Wqkv_i
        if bqkv_shards is not None and bqkv_shards[i] is not None:
            QKV = QKV + _f64(bqkv_shards[i])
        O_i = np.empty((M, n), dtype=F64)
        dQKV = np.empty((M, 3 * n), dtype=F64)
        dO_i = dY @ Wo_i.T
        for b in range(B):
            sl = slice(b * S, (b + 1) * S)
            q = QKV[sl, 0:n].reshape(S, Hg, d)
            k = QKV[sl, n:2 * n].reshape(S, Hg, d)
            v = QKV[sl, 2 * n:3 * n].reshape(S, Hg, d)
            O_i[sl] = attention_heads(q, k, v, causal).reshape(S, n)
            gq, gk, gv = attention_heads_backward(q, k, v, dO_i[sl].reshape(S, Hg, d), causal)
            dQKV[sl] = np.concatenate([gq.reshape(S, n), gk.reshape(S, n), gv.reshape(S, n)], axis=1)
        dWo.append(O_i.T @ dY)
        dWqkv.append(X.T @ dQKV)
        dbqkv.append(dQKV.sum(axis=0))
        part = dQKV @ Wqkv_i.T
        dX = part if dX is None else dX + part
    return dX, dWqkv, dbqkv, dWo, dY.sum(axis=0)
