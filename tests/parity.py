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
