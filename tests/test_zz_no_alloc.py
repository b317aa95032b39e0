"""The FFN entry point that allocates nothing (tp_ffn_forward_noalloc).

It serves callers that cannot give the library a workspace: code inside a host
framework that owns the whole device memory pool, or loops where a cudaMalloc
(and the device synchronisation it may imply) is not allowed.  Its act(Z)
scratch is a static 16 MiB device array in the library.  These tests call it
through the C ABI on two calls in a row and check that

* its output is bitwise equal to tp_ffn_forward's (caller workspace): both run
  the same two kernels on the same inputs, so a wrong scratch address, a stale
  read or a wrong stride would show as a bit difference;
* one call matches the fp64 oracle within the parity tolerance;
* a warm call changes the device's free memory by nothing;
* a call too large for the scratch is rejected.

The file is collected last on purpose.
"""
import pytest
import torch

from megatron_tensor_transformer_bias_b200 import inputs
from megatron_tensor_transformer_bias_b200 import tpblock as tb
from tests.parity import assert_bf16_close, ffn_oracle_rows

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _both(M, h, f, t, seed):
    p = inputs.ffn_inputs(M, h, f, "bf16", seed=seed, device=DEV)
    W1 = tb.shard_columns(p["W1"], t)
    W2 = tb.shard_rows(p["W2"], t)
    b1 = tb.shard_vector(p["b1"], t)
    ref = torch.empty_like(p["X"])
    tb.tp_ffn_forward(p["X"], W1, b1, W2, p["b2"], p["X"], ref)
    got = torch.empty_like(p["X"])
    tb.tp_ffn_forward_noalloc(p["X"], W1, b1, W2, p["b2"], p["X"], got)
    assert tb.tp_get_device_status() == tb.TP_OK
    return got, ref, p


def test_noalloc_matches_workspace_entry_point_two_calls_in_a_row():
    # two calls in a row on the shared static scratch, different shapes and inputs
    got, ref, p = _both(384, 512, 4096, 4, seed=31)
    assert torch.equal(got, ref), "no-alloc call 1 differs from tp_ffn_forward"
    rows = list(range(384))
    assert_bf16_close(got, ffn_oracle_rows(p, rows), "no-alloc call 1 vs oracle")
    got, ref, _ = _both(300, 256, 2048, 2, seed=32)   # ragged M; leaves stale data of call 1 past M*f
    assert torch.equal(got, ref), "no-alloc call 2 differs from tp_ffn_forward"


def test_noalloc_warm_call_leaves_free_memory_unchanged():
    M, h, f, t = 256, 256, 1024, 2
    p = inputs.ffn_inputs(M, h, f, "bf16", seed=34, device=DEV)
    W1, W2, b1 = tb.shard_columns(p["W1"], t), tb.shard_rows(p["W2"], t), tb.shard_vector(p["b1"], t)
    out = torch.empty_like(p["X"])
    tb.tp_ffn_forward_noalloc(p["X"], W1, b1, W2, p["b2"], p["X"], out)   # warm: module and symbol loaded
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        tb.tp_ffn_forward_noalloc(p["X"], W1, b1, W2, p["b2"], p["X"], out)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, f"free device memory moved by {free0 - free1} bytes"
    assert tb.tp_get_device_status() == tb.TP_OK


def test_noalloc_rejects_sizes_beyond_scratch():
    p = inputs.ffn_inputs(1024, 256, 8448, "bf16", seed=33, device=DEV)  # M*f = 8,650,752 > 8,388,608
    out = torch.empty_like(p["X"])
    with pytest.raises(tb.TPError) as e:
        tb.tp_ffn_forward_noalloc(p["X"], tb.shard_columns(p["W1"], 1), None, tb.shard_rows(p["W2"], 1), None,
                                  None, out)
    assert e.value.status == tb.TP_ERR_UNSUPPORTED
    assert "static scratch holds" in str(e.value)
