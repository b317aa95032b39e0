"""Seeded synthetic inputs shared by the CUDA path's tests, the bench and the oracle.

This module draws random numbers and lays them out; it computes nothing of the
block itself.  Each tensor has its own torch generator seeded with
``seed + OFFSET[name]``, drawn as fp32 ``randn * std`` on the requested device
and then rounded (round-to-nearest-even) to bf16 unless the workload is fp32.
The same call on the same device always returns the same bits.

Shard layout (the "i-th column shard" / "i-th row shard" of
"Tensor Parallelism > Combining Column and Row Parallelism", steps 1 and 2, read
as contiguous equal blocks):

* W1 ``[h, f]``: shard i is the column block ``[:, i*f/t:(i+1)*f/t]``.
* W2 ``[f, h]``: shard i is the row block ``[i*f/t:(i+1)*f/t, :]``.
* Wq, Wk, Wv ``[h, H*d]`` (head g at columns ``g*d..g*d+d``) are packed per
  head group into ``Wqkv [h, 3*H*d]``: shard i owns the column block
  ``[i*3*Hg*d, (i+1)*3*Hg*d)`` = ``[Q heads of group i | K heads | V heads]``.
* Wo ``[H*d, h]``: shard i is the row block of its heads.
"""
from __future__ import annotations

import torch

OFFSET = {
    "X": 0, "W1": 1, "b1": 2, "W2": 3, "b2": 4,
    "Wq": 5, "Wk": 6, "Wv": 7, "Wo": 8, "bo": 9,
    "rows": 100,
}
W_STD = 0.02
B_STD = 0.01


def _randn(shape, name, seed, device, std, dtype, offset_extra=0):
    g = torch.Generator(device=device)
    g.manual_seed(seed + OFFSET[name] + offset_extra)
    x = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


def _dt(dtype: str):
    return {"bf16": torch.bfloat16, "fp32": torch.float32}[dtype]


def ffn_inputs(M, h, f, dtype="bf16", seed=0, device="cpu", layer_offset=0):
    """X [M,h], W1 [h,f], b1 [f], W2 [f,h], b2 [h]; the residual is X."""
    dt = _dt(dtype)
    return {
        "X": _randn((M, h), "X", seed, device, 1.0, dt, layer_offset),
        "W1": _randn((h, f), "W1", seed, device, W_STD, dt, layer_offset),
        "b1": _randn((f,), "b1", seed, device, B_STD, dt, layer_offset),
        "W2": _randn((f, h), "W2", seed, device, W_STD, dt, layer_offset),
        "b2": _randn((h,), "b2", seed, device, B_STD, dt, layer_offset),
    }


def attn_inputs(B, S, h, H, d, seed=0, device="cpu", layer_offset=0):
    """X [B*S,h], Wq/Wk/Wv [h,H*d], Wo [H*d,h], bo [h] (bf16); the residual is X."""
    dt = torch.bfloat16
    return {
        "X": _randn((B * S, h), "X", seed, device, 1.0, dt, layer_offset),
        "Wq": _randn((h, H * d), "Wq", seed, device, W_STD, dt, layer_offset),
        "Wk": _randn((h, H * d), "Wk", seed, device, W_STD, dt, layer_offset),
        "Wv": _randn((h, H * d), "Wv", seed, device, W_STD, dt, layer_offset),
        "Wo": _randn((H * d, h), "Wo", seed, device, W_STD, dt, layer_offset),
        "bo": _randn((h,), "bo", seed, device, B_STD, dt, layer_offset),
    }


def layer_inputs(B, S, h, H, d, f, seed=0, device="cpu"):
    """Inputs of the pre-LN layer: attention weights, FFN weights, LayerNorm gamma=1, beta=0.

    The FFN tensors reuse the FFN offsets shifted by 1000 so that they differ
    from the attention tensors drawn from the same seed.
    """
    a = attn_inputs(B, S, h, H, d, seed, device)
    m = ffn_inputs(B * S, h, f, "bf16", seed, device, layer_offset=1000)
    out = dict(a)
    out.update({k: m[k] for k in ("W1", "b1", "W2", "b2")})
    one = torch.ones(h, dtype=torch.bfloat16, device=device)
    zero = torch.zeros(h, dtype=torch.bfloat16, device=device)
    out.update({"ln1_g": one, "ln1_b": zero, "ln2_g": one.clone(), "ln2_b": zero.clone()})
    return out


def pack_qkv(Wq, Wk, Wv, t, H, d):
    """Pack per-head Q/K/V weights into the head-group shard layout ``[h, 3*H*d]``."""
    assert H % t == 0
    Hg = H // t
    blocks = []
    for i in range(t):
        cols = slice(i * Hg * d, (i + 1) * Hg * d)
        blocks += [Wq[:, cols], Wk[:, cols], Wv[:, cols]]
    return torch.cat(blocks, dim=1).contiguous()


def sample_rows(M, n, seed=0, seq=None):
    """A seeded sample of ``n`` distinct token rows in ``[0, M)``, sorted.

    With ``seq`` given, the first and last token of every sequence are always
    included (causal attention's extreme cases).
    """
    n = min(n, M)
    must = []
    if seq is not None:
        for b in range(M // seq):
            must += [b * seq, b * seq + seq - 1]
    must = sorted(set(must))[:n]
    g = torch.Generator(device="cpu")
    g.manual_seed(seed + OFFSET["rows"])
    perm = torch.randperm(M, generator=g).tolist()
    chosen = list(must)
    seen = set(must)
    for r in perm:
        if len(chosen) >= n:
            break
        if r not in seen:
            chosen.append(r)
            seen.add(r)
    return sorted(chosen)


def as_fp16(w):
    """An fp16 copy of a bf16 weight (same values: bf16 -> fp16 is exact for every
    |w| >= 2**-17 below 65504, which covers N(0, 0.02^2) weights but for about
    3 in 10^4 entries, whose change is below 2**-25 in absolute value)."""
    return w.to(torch.float16)
