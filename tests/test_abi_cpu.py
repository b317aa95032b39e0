"""The C-ABI library loads, exports what include/tpblock.h declares, and its host
validation rejects bad arguments before any launch (CPU only: every call here
fails validation or does no device work, so no GPU is touched)."""
import ctypes
import os
import re

import pytest

from megatron_tensor_transformer_bias_b200 import tpblock as tb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tpblock.h")


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^TP_API\s+[\w\s\*]+?\b(tp_\w+)\(", src, flags=re.M)))


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(tb.LIB_PATH):
        from megatron_tensor_transformer_bias_b200 import build
        build.build()
    return tb.lib()


def test_every_declared_symbol_is_exported(L):
    names = _declared()
    assert len(names) >= 20
    for n in names:
        assert hasattr(L, n), n
    # and the binding declares a signature for each
    assert set(names) == set(tb._SIGS), set(names) ^ set(tb._SIGS)


def test_version_and_status_strings(L):
    assert L.tp_version() == 1
    assert tb.status_string(tb.TP_OK) == "TP_OK"
    assert tb.status_string(tb.TP_ERR_TIMEOUT) == "TP_ERR_TIMEOUT"
    assert tb.status_string(99) == "TP_ERR_UNKNOWN"


def test_workspace_sizes(L):
    M, h, f, t = 2048, 4096, 16384, 4
    z = M * f * 2
    assert tb.tp_ffn_workspace_bytes(M, h, f, t, tb.TP_BF16, tb.TP_REDUCE_FUSED) == z
    ctr = ((M + 31) // 32) * ((h + 127) // 128) * 4          # arrival counters of the in-epilogue reduction
    assert tb.tp_ffn_workspace_bytes(M, h, f, t, tb.TP_BF16, tb.TP_REDUCE_PARTIALS) == z + t * M * h * 4 + ctr
    assert tb.tp_ffn_workspace_bytes(8, 64, 256, 2, tb.TP_FP32, tb.TP_REDUCE_FUSED) == 8 * 256 * 4 + 2 * 8 * 64 * 4
    assert tb.tp_ffn_workspace_bytes(0, h, f, t) == 0
    assert L.tp_row_linear_workspace_bytes(M, h, t, tb.TP_REDUCE_FUSED) == 0
    assert L.tp_row_linear_workspace_bytes(M, h, t, tb.TP_REDUCE_PARTIALS) == t * M * h * 4 + ctr
    mf = M * f * 2
    assert tb.tp_ffn_backward_workspace_bytes(M, h, f, t) == 3 * mf   # act(Z), act'(Z), dZ
    assert tb.tp_ffn_backward_workspace_bytes(0, h, f, t) == 0
    B, S, H, d = 2, 2048, 32, 128
    q = B * S * H * d * 2
    assert tb.tp_attn_workspace_bytes(B, S, 4096, H, d, 4, tb.TP_REDUCE_FUSED) == 4 * q
    assert tb.tp_layer_workspace_bytes(1, 2048, 8192, 64, 128, 32768, 8) > 2048 * 32768 * 2


# ---------------------------------------------------------------- host validation
FAKE = 1 << 20  # a 16-byte-aligned non-null address; never dereferenced (validation fails first)


def _sh(t, ld, base=FAKE, step=1 << 16):
    arr = (tb.Shard * t)()
    for i in range(t):
        arr[i].ptr = base + i * step
        arr[i].ld = ld
    return arr


def _ffn(L, M=256, h=256, f=1024, t=2, X=FAKE, out=FAKE + 4096, W1=None, W2=None, b2=None, res=None,
         dtype=tb.TP_BF16, mode=tb.TP_REDUCE_FUSED, act=tb.TP_ACT_GELU, ws=FAKE, ws_bytes=0):
    W1 = _sh(t, f) if W1 is None else W1
    W2 = _sh(t, h) if W2 is None else W2
    return L.tp_ffn_forward_act(X, M, h, f, t, W1, None, W2, b2, res, out, dtype, mode, act, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,code,msg", [
    (dict(X=None), tb.TP_ERR_INVALID_ARG, "X is NULL"),
    (dict(out=None), tb.TP_ERR_INVALID_ARG, "out is NULL"),
    (dict(X=FAKE + 8), tb.TP_ERR_INVALID_ARG, "16-byte"),
    (dict(t=0), tb.TP_ERR_INVALID_ARG, "t=0"),
    (dict(t=17), tb.TP_ERR_INVALID_ARG, "t=17"),
    (dict(f=1000, t=3), tb.TP_ERR_INVALID_ARG, "not divisible"),
    (dict(h=200), tb.TP_ERR_UNSUPPORTED, "h % 64"),
    (dict(f=96, t=1), tb.TP_ERR_UNSUPPORTED, "(f/t) % 64"),
    (dict(M=-1), tb.TP_ERR_INVALID_ARG, "positive"),
    (dict(dtype=7), tb.TP_ERR_INVALID_ARG, "dtype"),
    (dict(mode=5), tb.TP_ERR_INVALID_ARG, "mode"),
    (dict(act=9), tb.TP_ERR_INVALID_ARG, "activation"),
    (dict(out=FAKE), tb.TP_ERR_INVALID_ARG, "alias"),
    (dict(), tb.TP_ERR_WORKSPACE, "workspace"),
])
def test_ffn_validation(L, kw, code, msg):
    s = _ffn(L, **kw)
    assert s == code, (tb.status_string(s), tb.last_error())
    assert msg in tb.last_error()


def test_ffn_shard_validation(L):
    assert _ffn(L, W1=_sh(2, 100)) == tb.TP_ERR_INVALID_ARG and "ld" in tb.last_error()   # ld < cols... or %8
    assert _ffn(L, W1=_sh(2, 1028)) == tb.TP_ERR_INVALID_ARG and "multiple of 8" in tb.last_error()
    bad = _sh(2, 1024)
    bad[1].ptr = 0
    assert _ffn(L, W1=bad) == tb.TP_ERR_INVALID_ARG and "W1[1].ptr is NULL" in tb.last_error()
    bad = _sh(2, 256)
    bad[0].ptr = FAKE + 2
    assert _ffn(L, W2=bad) == tb.TP_ERR_INVALID_ARG and "W2[0]" in tb.last_error()


def test_shard_dtype_validation(L):
    bad = _sh(2, 1024)
    bad[1].dtype = tb.TP_FP16
    assert _ffn(L, W1=bad) == tb.TP_ERR_INVALID_ARG and "mix" in tb.last_error()
    bad = _sh(2, 1024)
    bad[0].dtype = bad[1].dtype = 7
    assert _ffn(L, W1=bad) == tb.TP_ERR_INVALID_ARG and "dtype" in tb.last_error()
    f16 = _sh(2, 1024)
    f16[0].dtype = f16[1].dtype = tb.TP_FP16
    assert _ffn(L, W1=f16) == tb.TP_ERR_INVALID_ARG and "W1 must have X's dtype" in tb.last_error()
    w2 = _sh(2, 256)
    w2[0].dtype = w2[1].dtype = tb.TP_FP16
    assert _ffn(L, W2=w2) == tb.TP_ERR_WORKSPACE  # fp16 W2 is valid: fails only on the missing workspace


def test_ffn_empty_is_ok_without_launch(L):
    # M = 0: valid, nothing to do, no device touched
    assert _ffn(L, M=0, ws=None) == tb.TP_OK


def test_attention_validation(L):
    t = 2
    Wqkv = _sh(t, 3 * 2 * 128)
    Wo = _sh(t, 256)
    call = lambda **k: L.tp_attn_forward(k.get("X", FAKE), k.get("B", 1), k.get("S", 64), k.get("h", 256),
                                         k.get("H", 4), k.get("d", 128), k.get("t", t), k.get("Wqkv", Wqkv), None,
                                         Wo, None, None, 1, k.get("out", FAKE + 4096), 0, FAKE, 0, None)
    assert call(d=64) == tb.TP_ERR_UNSUPPORTED and "head dim" in tb.last_error()
    assert call(H=3) == tb.TP_ERR_INVALID_ARG and "divisible" in tb.last_error()
    assert call(X=None) == tb.TP_ERR_INVALID_ARG
    assert call() == tb.TP_ERR_WORKSPACE
    assert call(B=0) == tb.TP_OK
    f16 = _sh(t, 3 * 2 * 128)
    f16[0].dtype = f16[1].dtype = tb.TP_FP16
    assert call(Wqkv=f16) == tb.TP_ERR_INVALID_ARG and "Wqkv must have X's dtype" in tb.last_error()


def test_layer_and_building_block_validation(L):
    assert L.tp_layernorm_forward(FAKE, 0, None, None, 4, 100, 1e-5, FAKE + 4096, 0, None) == tb.TP_ERR_UNSUPPORTED
    assert L.tp_layernorm_forward(FAKE, 0, None, None, 4, 128, 0.0, FAKE + 4096, 0, None) == tb.TP_ERR_INVALID_ARG
    assert L.tp_layernorm_forward(None, 0, None, None, 4, 128, 1e-5, FAKE, 0, None) == tb.TP_ERR_INVALID_ARG
    assert L.tp_layernorm_forward(FAKE, 0, None, None, 4, 128, 1e-5, FAKE, 1, None) == tb.TP_ERR_INVALID_ARG
    assert L.tp_reduce_partials(FAKE, 0, 4, 128, None, None, 0, FAKE, None) == tb.TP_ERR_INVALID_ARG
    assert L.tp_reduce_partials(FAKE, 2, 4, 126, None, None, 0, FAKE, None) == tb.TP_ERR_UNSUPPORTED
    assert L.tp_selftest_bounded_wait(0, None) == tb.TP_ERR_INVALID_ARG
    assert L.tp_activation_forward(None, FAKE, 10, 0, None) == tb.TP_ERR_INVALID_ARG
    assert L.tp_activation_forward(FAKE, FAKE, 10, 7, None) == tb.TP_ERR_INVALID_ARG
    assert L.tp_activation_forward(FAKE, FAKE, -1, 0, None) == tb.TP_ERR_INVALID_ARG
    assert L.tp_activation_forward(None, None, 0, 0, None) == tb.TP_OK
    assert L.tp_trace_enable(0) == tb.TP_ERR_INVALID_ARG
    assert L.tp_column_linear_forward(FAKE, 4, 100, 128, 1, _sh(1, 128), None, -1, FAKE, None) == tb.TP_ERR_UNSUPPORTED
    assert L.tp_row_linear_forward(FAKE, 4, 128, 128, 1, _sh(1, 128), None, None, FAKE + 4096, 1, None, 0,
                                   None) == tb.TP_ERR_WORKSPACE


def test_binding_requires_library(monkeypatch):
    monkeypatch.setattr(tb, "_lib", None)
    monkeypatch.setattr(tb, "LIB_PATH", "/nonexistent/libtpblock.so")
    with pytest.raises(RuntimeError, match="not built"):
        tb.lib()


def test_backward_validation(L):
    M, h, f, t = 256, 256, 1024, 2

    def call(**k):
        return L.tp_ffn_backward(k.get("X", FAKE), k.get("M", M), h, k.get("f", f), t, k.get("W1", _sh(t, f)), None,
                                 k.get("W2", _sh(t, h)), k.get("dY", FAKE + 8192), None, k.get("dX", FAKE + 4096),
                                 k.get("dW1", FAKE + 16384), None, k.get("dW2", FAKE + 32768), None,
                                 k.get("act", tb.TP_ACT_GELU), k.get("ws", FAKE), 0, None)
    assert call(dY=None) == tb.TP_ERR_INVALID_ARG and "dY is NULL" in tb.last_error()
    assert call(dW1=None) == tb.TP_ERR_INVALID_ARG and "dW1 is NULL" in tb.last_error()
    assert call(dX=FAKE) == tb.TP_ERR_INVALID_ARG and "alias" in tb.last_error()
    assert call(act=5) == tb.TP_ERR_INVALID_ARG and "activation" in tb.last_error()
    assert call(f=1001) == tb.TP_ERR_INVALID_ARG and "divisible" in tb.last_error()
    w2 = _sh(t, h)
    w2[0].dtype = w2[1].dtype = tb.TP_FP16
    assert call(W2=w2) == tb.TP_ERR_UNSUPPORTED and "bf16" in tb.last_error()
    assert call() == tb.TP_ERR_WORKSPACE and "workspace" in tb.last_error()


def test_attn_backward_workspace_and_validation(L):
    B, S, h, H, d, t = 2, 2048, 4096, 32, 128, 4
    q = B * S * H * d * 2
    vec = B * H * 2048 * 4
    assert tb.tp_attn_backward_workspace_bytes(B, S, h, H, d, t) == 8 * q + 2 * vec
    assert tb.tp_attn_backward_workspace_bytes(0, S, h, H, d, t) == 0
    # S not a multiple of 128: the row vectors are padded to whole 128-query blocks
    assert tb.tp_attn_backward_workspace_bytes(1, 200, 256, 2, d, 1) >= 8 * (200 * 2 * d * 2) + 2 * 2 * 256 * 4

    Bs, Ss, hs, Hs, ts = 1, 128, 256, 2, 2
    n = (Hs // ts) * d

    def call(**k):
        return L.tp_attn_backward(k.get("X", FAKE), Bs, Ss, hs, Hs, k.get("d", d), ts, k.get("Wqkv", _sh(ts, 3 * n)),
                                  None, k.get("Wo", _sh(ts, hs)), k.get("dY", FAKE + 8192), None, 1,
                                  k.get("dX", FAKE + 4096), k.get("dWqkv", FAKE + 16384), None,
                                  k.get("dWo", FAKE + 32768), None, k.get("ws", FAKE), 0, None)
    assert call(dY=None) == tb.TP_ERR_INVALID_ARG and "dY is NULL" in tb.last_error()
    assert call(dWqkv=None) == tb.TP_ERR_INVALID_ARG and "dWqkv is NULL" in tb.last_error()
    assert call(dWo=None) == tb.TP_ERR_INVALID_ARG and "dWo is NULL" in tb.last_error()
    assert call(dX=FAKE) == tb.TP_ERR_INVALID_ARG and "alias" in tb.last_error()
    assert call(d=64) == tb.TP_ERR_UNSUPPORTED and "d=64" in tb.last_error()
    wo = _sh(ts, hs)
    wo[0].dtype = wo[1].dtype = tb.TP_FP16
    assert call(Wo=wo) == tb.TP_ERR_UNSUPPORTED and "bf16" in tb.last_error()
    assert call() == tb.TP_ERR_WORKSPACE and "workspace" in tb.last_error()
