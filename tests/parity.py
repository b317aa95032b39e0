"""Tolerances and helpers shared by the GPU parity tests.

bf16 workloads: relative Frobenius error <= 5e-3 and, element by element,
|gpu - ref| <= 3e-2 + 2e-2 * |ref|.  fp32 workload: relative Frobenius error
<= 1e-5.  The reference is always the fp64 oracle on the same input bits.
"""
import numpy as np
import torch

import oracle

BF16_REL_FRO = 5e-3
BF16_ABS = 3e-2
BF16_REL = 2e-2
FP32_REL_FRO = 1e-5


def to64(t):
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu", torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


def errors(got, ref):
    got, ref = to64(got), to64(ref)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), "non-finite GPU output"
    diff = got - ref
    rel_fro = float(np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-300))
    excess = np.abs(diff) - (BF16_ABS + BF16_REL * np.abs(ref))
    return rel_fro, float(excess.max()), float(np.abs(diff).max())


def assert_bf16_close(got, ref, what=""):
    rel_fro, excess, maxabs = errors(got, ref)
    assert rel_fro <= BF16_REL_FRO, f"{what}: rel Frobenius {rel_fro:.3e} > {BF16_REL_FRO}"
    assert excess <= 0, f"{what}: element error above 3e-2 + 2e-2|ref| (max |err| {maxabs:.3e})"
    return rel_fro


def assert_fp32_close(got, ref, what=""):
    got, ref = to64(got), to64(ref)
    rel = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
    assert rel <= FP32_REL_FRO, f"{what}: rel Frobenius {rel:.3e} > {FP32_REL_FRO}"
    return rel


def ffn_oracle_rows(inp, rows, chunks=8, act="gelu"):
    """Oracle FFN output at the given token rows, streaming W1/W2 in column/row
    chunks (the sharded form of the block, which equals the plain block)."""
    X, W1, b1, W2, b2 = inp["X"], inp["W1"], inp["b1"], inp["W2"], inp["b2"]
    f = W1.shape[1]
    while f % chunks:
        chunks //= 2
    n = f // chunks
    Xr = to64(X[rows])

    def shards():
        for i in range(chunks):
            cols = slice(i * n, (i + 1) * n)
            yield to64(W1[:, cols]), to64(b1[cols]), to64(W2[cols, :])

    return oracle.ffn_forward_sharded(Xr, shards(), to64(b2), Xr, act=act)


# ---------------------------------------------------------------- gradients
# The backward pass's outputs are sums of products one factor of which was rounded to a
# 16-bit type before the sum: dW1 = X^T dZ and db1 = sum dZ (dZ stored in bf16 after a
# multiplication by act'(Z) stored in fp16), dW2 = A^T dY (A = act(Z) stored in bf16),
# dX = dZ W1^T (+ dY, then rounded to bf16).  With u = 2^-8, bf16's unit roundoff, each
# rounded factor carries a relative error |delta_k| <= 1.125 u (bf16 plus fp16), so an
# element sum_k a_k b_k (1 + delta_k) is off by sum_k a_k b_k delta_k: independent
# roundings give a standard deviation below 0.65 u * sqrt(sum_k (a_k b_k)^2).  The bound is
# 6 u times that root-sum-square ("scale", > 9 standard deviations) plus u |ref| for a
# gradient stored in bf16, and the relative Frobenius error must stay within the forward
# pass's 5e-3.  fp32 accumulation (2^-24 per add) is far below both.
BF16_U = 2.0 ** -8
GRAD_SIGMAS = 6.0


def assert_grad_close(got, ref, scale, what="", bf16_out=False):
    got, ref, scale = to64(got), to64(ref), to64(scale)
    assert got.shape == ref.shape == scale.shape, (got.shape, ref.shape, scale.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite GPU output"
    diff = np.abs(got - ref)
    rel_fro = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))
    assert rel_fro <= BF16_REL_FRO, f"{what}: rel Frobenius {rel_fro:.3e} > {BF16_REL_FRO}"
    bound = GRAD_SIGMAS * BF16_U * scale + (BF16_U * np.abs(ref) if bf16_out else 0.0) + 1e-6 * np.abs(ref).max()
    worst = float((diff / bound).max())
    assert worst <= 1.0, f"{what}: element error {worst:.2f}x the bound (max |err| {diff.max():.3e})"
    return rel_fro


def grad_scales(X, W1, b1, W2, dY, act="gelu"):
    """Root-sum-squares of the products behind each gradient element (fp64, for the bound)."""
    X, W1, W2, dY = to64(X), to64(W1), to64(W2), to64(dY)
    Z = X @ W1
    if b1 is not None:
        Z = Z + to64(b1)
    A = oracle.gelu(Z) if act == "gelu" else oracle.relu(Z)
    dZ = (dY @ W2.T) * (oracle.gelu_grad(Z) if act == "gelu" else oracle.relu_grad(Z))
    return {"dX": np.sqrt((dZ ** 2) @ (W1 ** 2).T), "dW1": np.sqrt((X ** 2).T @ (dZ ** 2)),
            "db1": np.sqrt((dZ ** 2).sum(axis=0)), "dW2": np.sqrt((A ** 2).T @ (dY ** 2)),
            "db2": np.sqrt((dY ** 2).sum(axis=0))}
