"""The FFN entry point that allocates nothing (tp_ffn_forward_noalloc).

It serves callers that cannot give the library a workspace: code inside a host
framework that owns the whole device memory pool, or loops where a cudaMalloc
(and the device synchronisation it may imply) is not allowed.  Its act(Z)
scratch is a static 16 MiB device array in the library.  These tests call it
through the C ABI and compare it with tp_ffn_forward (caller workspace) within
the parity tolerance, on two calls in a row, and check that a call too large
for the scratch is rejected.  The file is collected last on purpose.
"""
import pytest
import torch

from megatron_tensor_transformer_bias_b200 import inputs
from megatron_tensor_transformer_bias_b200 import tpblock as tb
from tests.parity import assert_bf16_close

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
    return got, ref


def test_noalloc_matches_workspace_entry_point_two_calls_in_a_row():
    # two calls in a row on the shared static scratch, different shapes and inputs
    got, ref = _both(384, 512, 4096, 4, seed=31)
    assert_bf16_close(got, ref, "no-alloc call 1")
    got, ref = _both(300, 256, 2048, 2, seed=32)   # ragged M; leaves stale data of call 1 past M*f
    assert_bf16_close(got, ref, "no-alloc call 2")


def test_noalloc_rejects_sizes_beyond_scratch():
    p = inputs.ffn_inputs(1024, 256, 8448, "bf16", seed=33, device=DEV)  # M*f = 8,650,752 > 8,388,608
    out = torch.empty_like(p["X"])
    with pytest.raises(tb.TPError) as e:
        tb.tp_ffn_forward_noalloc(p["X"], tb.shard_columns(p["W1"], 1), None, tb.shard_rows(p["W2"], 1), None,
                                  None, out)
    assert e.value.status == tb.TP_ERR_UNSUPPORTED
    assert "static scratch holds" in str(e.value)
