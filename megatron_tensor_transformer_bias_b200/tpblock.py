"""Thin ctypes binding of libtpblock (``include/tpblock.h``): argument marshalling only.

Every function here takes torch tensors (device memory that torch allocated),
turns them into pointers, sizes and strides, and calls the C entry point of the
same name.  Nothing of the block is computed in Python; there is no CPU path.
If ``libtpblock.so`` is missing, the first call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import List, Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtpblock.so")

TP_OK, TP_ERR_INVALID_ARG, TP_ERR_UNSUPPORTED, TP_ERR_WORKSPACE, TP_ERR_CUDA, TP_ERR_TIMEOUT, TP_ERR_RANGE = range(7)
TP_BF16, TP_FP32, TP_FP16 = 0, 1, 2
TP_REDUCE_FUSED, TP_REDUCE_PARTIALS = 0, 1
TP_ACT_GELU, TP_ACT_RELU = 0, 1
TP_MAX_SHARDS = 16

MODES = {"fused": TP_REDUCE_FUSED, "partials": TP_REDUCE_PARTIALS}
ACTS = {"gelu": TP_ACT_GELU, "relu": TP_ACT_RELU, None: -1, "none": -1}


class Shard(ctypes.Structure):
    _fields_ = [("ptr", ctypes.c_void_p), ("ld", ctypes.c_int64), ("dtype", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


class TPError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{status_string(status)}: {msg}")
        self.status = status


_lib = None
_vp, _i64, _i32, _sz, _f32, _u64 = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t,
                                    ctypes.c_float, ctypes.c_uint64)
_SP = ctypes.POINTER(Shard)
_VPP = ctypes.POINTER(ctypes.c_void_p)

_SIGS = {
    "tp_ffn_workspace_bytes": (_sz, [_i64, _i64, _i64, _i32, _i32, _i32]),
    "tp_ffn_forward": (_i32, [_vp, _i64, _i64, _i64, _i32, _SP, _VPP, _SP, _vp, _vp, _vp, _i32, _i32, _vp, _sz, _vp]),
    "tp_ffn_forward_act": (_i32, [_vp, _i64, _i64, _i64, _i32, _SP, _VPP, _SP, _vp, _vp, _vp, _i32, _i32, _i32, _vp,
                                  _sz, _vp]),
    "tp_ffn_forward_noalloc": (_i32, [_vp, _i64, _i64, _i64, _i32, _SP, _VPP, _SP, _vp, _vp, _vp, _vp]),
    "tp_ffn_backward_workspace_bytes": (_sz, [_i64, _i64, _i64, _i32]),
    "tp_ffn_backward": (_i32, [_vp, _i64, _i64, _i64, _i32, _SP, _VPP, _SP, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32,
                               _vp, _sz, _vp]),
    "tp_column_linear_forward": (_i32, [_vp, _i64, _i64, _i64, _i32, _SP, _VPP, _i32, _vp, _vp]),
    "tp_row_linear_workspace_bytes": (_sz, [_i64, _i64, _i32, _i32]),
    "tp_row_linear_forward": (_i32, [_vp, _i64, _i64, _i64, _i32, _SP, _vp, _vp, _vp, _i32, _vp, _sz, _vp]),
    "tp_attn_workspace_bytes": (_sz, [_i32, _i32, _i32, _i32, _i32, _i32, _i32]),
    "tp_attn_forward": (_i32, [_vp, _i32, _i32, _i32, _i32, _i32, _i32, _SP, _VPP, _SP, _vp, _vp, _i32, _vp, _i32,
                               _vp, _sz, _vp]),
    "tp_attn_backward_workspace_bytes": (_sz, [_i32, _i32, _i32, _i32, _i32, _i32]),
    "tp_attn_backward": (_i32, [_vp, _i32, _i32, _i32, _i32, _i32, _i32, _SP, _VPP, _SP, _vp, _vp, _i32, _vp, _vp,
                                _vp, _vp, _vp, _vp, _sz, _vp]),
    "tp_layer_workspace_bytes": (_sz, [_i32, _i32, _i32, _i32, _i32, _i64, _i32, _i32]),
    "tp_layer_forward": (_i32, [_vp, _i32, _i32, _i32, _i32, _i32, _i64, _i32, _vp, _vp, _SP, _VPP, _SP, _vp, _vp,
                                _vp, _SP, _VPP, _SP, _vp, _f32, _i32, _vp, _i32, _vp, _sz, _vp]),
    "tp_layernorm_forward": (_i32, [_vp, _i32, _vp, _vp, _i64, _i64, _f32, _vp, _i32, _vp]),
    "tp_reduce_partials": (_i32, [_vp, _i32, _i64, _i64, _vp, _vp, _i32, _vp, _vp]),
    "tp_activation_forward": (_i32, [_vp, _vp, _i64, _i32, _vp]),
    "tp_get_device_status": (_i32, [_vp]),
    "tp_set_wait_limit_ns": (None, [_u64]),
    "tp_selftest_bounded_wait": (_i32, [_u64, _vp]),
    "tp_trace_enable": (_i32, [_i32]),
    "tp_trace_disable": (None, []),
    "tp_trace_count": (_i32, []),
    "tp_trace_get": (_i32, [_i32, ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(ctypes.c_float)]),
    "tp_status_string": (ctypes.c_char_p, [_i32]),
    "tp_last_error": (ctypes.c_char_p, []),
    "tp_version": (_i32, []),
}


def lib():
    """Load libtpblock.so (once) and declare every entry point's signature."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libtpblock.so is not built ({LIB_PATH}); run "
                               "`python -m megatron_tensor_transformer_bias_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def status_string(s: int) -> str:
    return lib().tp_status_string(s).decode()


def last_error() -> str:
    return lib().tp_last_error().decode()


def _check(s: int):
    if s != TP_OK:
        raise TPError(s, last_error())


# ---------------------------------------------------------------- marshalling
def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dev(t: torch.Tensor):
    if not t.is_cuda:
        raise ValueError("libtpblock takes CUDA tensors")
    return t


def _shards(ws: Sequence[torch.Tensor]):
    arr = (Shard * len(ws))()
    for i, w in enumerate(ws):
        _dev(w)
        if w.dim() != 2 or w.stride(1) != 1:
            raise ValueError("a shard must be a 2-D view with unit column stride")
        arr[i].ptr = w.data_ptr()
        arr[i].ld = w.stride(0)
        arr[i].dtype = TP_FP16 if w.dtype == torch.float16 else TP_BF16
    return arr


def _ptr_array(bs: Optional[Sequence[Optional[torch.Tensor]]]):
    if bs is None:
        return None
    arr = (ctypes.c_void_p * len(bs))()
    for i, b in enumerate(bs):
        arr[i] = None if b is None else _dev(b).data_ptr()
    return arr


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return TP_BF16
    if t.dtype == torch.float32:
        return TP_FP32
    if t.dtype == torch.float16:
        return TP_FP16
    raise ValueError(f"unsupported dtype {t.dtype}")


def workspace(nbytes: int, device) -> torch.Tensor:
    """Caller-owned device workspace (torch allocates it; the library never does)."""
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)


def shard_columns(W: torch.Tensor, t: int) -> List[torch.Tensor]:
    """Column shard views W[:, i*n/t:(i+1)*n/t] (no copies)."""
    n = W.shape[1] // t
    return [W[:, i * n:(i + 1) * n] for i in range(t)]


def shard_rows(W: torch.Tensor, t: int) -> List[torch.Tensor]:
    """Row shard views W[i*k/t:(i+1)*k/t, :] (no copies)."""
    k = W.shape[0] // t
    return [W[i * k:(i + 1) * k, :] for i in range(t)]


def shard_vector(b: Optional[torch.Tensor], t: int):
    if b is None:
        return None
    n = b.shape[0] // t
    return [b[i * n:(i + 1) * n] for i in range(t)]


# ---------------------------------------------------------------- FFN block
def tp_ffn_workspace_bytes(M, h, f, t, dtype=TP_BF16, mode=TP_REDUCE_FUSED) -> int:
    return lib().tp_ffn_workspace_bytes(M, h, f, t, dtype, mode)


def tp_ffn_forward(X, W1, b1, W2, b2, residual, out, mode="fused", act="gelu", ws=None, stream=None):
    """out = sum_i act(X W1[i] + b1[i]) W2[i] + b2 + residual (t = len(W1) shards)."""
    _dev(X); _dev(out)
    M, h = X.shape
    t = len(W1)
    f = sum(w.shape[1] for w in W1)
    dt = _dtype_code(X)
    m = MODES[mode] if isinstance(mode, str) else mode
    need = tp_ffn_workspace_bytes(M, h, f, t, dt, m)
    if ws is None:
        ws = workspace(need, X.device)
    s = lib().tp_ffn_forward_act(_ptr(X), M, h, f, t, _shards(W1), _ptr_array(b1), _shards(W2), _ptr(b2),
                                 _ptr(residual), _ptr(out), dt, m, ACTS[act], _ptr(ws), ws.numel(), _stream(stream))
    _check(s)
    return out


def tp_ffn_forward_noalloc(X, W1, b1, W2, b2, residual, out, stream=None):
    """The FFN block (GeLU, bf16, fused reduction) with act(Z) in the library's static
    16 MiB device scratch instead of a workspace, for callers that cannot allocate."""
    _dev(X); _dev(out)
    M, h = X.shape
    t = len(W1)
    f = sum(w.shape[1] for w in W1)
    _check(lib().tp_ffn_forward_noalloc(_ptr(X), M, h, f, t, _shards(W1), _ptr_array(b1), _shards(W2), _ptr(b2),
                                        _ptr(residual), _ptr(out), _stream(stream)))
    return out


def tp_ffn_backward_workspace_bytes(M, h, f, t) -> int:
    return lib().tp_ffn_backward_workspace_bytes(M, h, f, t)


def tp_ffn_backward(X, W1, b1, W2, dY, dX, dW1, dW2, db1=None, db2=None, dX_add=None, act="gelu", ws=None,
                    stream=None):
    """Gradients of the FFN block (bf16): dX [M,h] bf16, dW1 [h,f] fp32, dW2 [f,h] fp32,
    db1 [f] and db2 [h] fp32 (optional), for the upstream gradient dY [M,h] bf16."""
    for t_ in (X, dY, dX, dW1, dW2):
        _dev(t_)
    M, h = X.shape
    t = len(W1)
    f = sum(w.shape[1] for w in W1)
    if dW1.dtype != torch.float32 or dW2.dtype != torch.float32:
        raise ValueError("weight gradients are fp32")
    if ws is None:
        ws = workspace(tp_ffn_backward_workspace_bytes(M, h, f, t), X.device)
    _check(lib().tp_ffn_backward(_ptr(X), M, h, f, t, _shards(W1), _ptr_array(b1), _shards(W2), _ptr(dY),
                                 _ptr(dX_add), _ptr(dX), _ptr(dW1), _ptr(db1), _ptr(dW2), _ptr(db2), ACTS[act],
                                 _ptr(ws), ws.numel(), _stream(stream)))
    return dX, dW1, dW2, db1, db2


def tp_column_linear_forward(X, W, b, out, act=None, stream=None):
    M, k = X.shape
    t = len(W)
    n = sum(w.shape[1] for w in W)
    _check(lib().tp_column_linear_forward(_ptr(_dev(X)), M, k, n, t, _shards(W), _ptr_array(b), ACTS[act],
                                          _ptr(_dev(out)), _stream(stream)))
    return out


def tp_row_linear_forward(A, W, bias, residual, out, mode="fused", ws=None, stream=None):
    M, k = A.shape
    t = len(W)
    n = W[0].shape[1]
    m = MODES[mode] if isinstance(mode, str) else mode
    need = lib().tp_row_linear_workspace_bytes(M, n, t, m)
    if ws is None and need:
        ws = workspace(need, A.device)
    _check(lib().tp_row_linear_forward(_ptr(_dev(A)), M, k, n, t, _shards(W), _ptr(bias), _ptr(residual),
                                       _ptr(_dev(out)), m, _ptr(ws), 0 if ws is None else ws.numel(),
                                       _stream(stream)))
    return out


# ---------------------------------------------------------------- attention / layer
def tp_attn_workspace_bytes(B, S, h, heads, d, t, mode=TP_REDUCE_FUSED) -> int:
    return lib().tp_attn_workspace_bytes(B, S, h, heads, d, t, mode)


def tp_attn_forward(X, B, S, heads, d, Wqkv, bqkv, Wo, bo, residual, out, causal=True, mode="fused", ws=None,
                    stream=None):
    _dev(X); _dev(out)
    h = X.shape[1]
    t = len(Wqkv)
    m = MODES[mode] if isinstance(mode, str) else mode
    if ws is None:
        ws = workspace(tp_attn_workspace_bytes(B, S, h, heads, d, t, m), X.device)
    _check(lib().tp_attn_forward(_ptr(X), B, S, h, heads, d, t, _shards(Wqkv), _ptr_array(bqkv), _shards(Wo),
                                 _ptr(bo), _ptr(residual), 1 if causal else 0, _ptr(out), m, _ptr(ws), ws.numel(),
                                 _stream(stream)))
    return out


def tp_attn_backward_workspace_bytes(B, S, h, heads, d, t) -> int:
    return lib().tp_attn_backward_workspace_bytes(B, S, h, heads, d, t)


def tp_attn_backward(X, B, S, heads, d, Wqkv, bqkv, Wo, dY, dX, dWqkv, dWo, dbqkv=None, dbo=None, dX_add=None,
                     causal=True, ws=None, stream=None):
    """Gradients of the attention sub-layer (bf16): dX [B*S,h] bf16, dWqkv [h, 3*heads*d] fp32
    (group i's [Q|K|V] column block i), dWo [heads*d, h] fp32, dbqkv [3*heads*d] and dbo [h]
    fp32 (optional), for the upstream gradient dY [B*S,h] bf16."""
    for t_ in (X, dY, dX, dWqkv, dWo):
        _dev(t_)
    h = X.shape[1]
    t = len(Wqkv)
    if dWqkv.dtype != torch.float32 or dWo.dtype != torch.float32:
        raise ValueError("weight gradients are fp32")
    if ws is None:
        ws = workspace(tp_attn_backward_workspace_bytes(B, S, h, heads, d, t), X.device)
    _check(lib().tp_attn_backward(_ptr(X), B, S, h, heads, d, t, _shards(Wqkv), _ptr_array(bqkv), _shards(Wo),
                                  _ptr(dY), _ptr(dX_add), 1 if causal else 0, _ptr(dX), _ptr(dWqkv), _ptr(dbqkv),
                                  _ptr(dWo), _ptr(dbo), _ptr(ws), ws.numel(), _stream(stream)))
    return dX, dWqkv, dWo, dbqkv, dbo


def tp_layer_workspace_bytes(B, S, h, heads, d, f, t, mode=TP_REDUCE_FUSED) -> int:
    return lib().tp_layer_workspace_bytes(B, S, h, heads, d, f, t, mode)


def tp_layer_forward(X, B, S, heads, d, ln1_g, ln1_b, Wqkv, bqkv, Wo, bo, ln2_g, ln2_b, W1, b1, W2, b2, out,
                     eps=1e-5, causal=True, mode="fused", ws=None, stream=None):
    _dev(X); _dev(out)
    h = X.shape[1]
    t = len(Wqkv)
    f = sum(w.shape[1] for w in W1)
    m = MODES[mode] if isinstance(mode, str) else mode
    if ws is None:
        ws = workspace(tp_layer_workspace_bytes(B, S, h, heads, d, f, t, m), X.device)
    _check(lib().tp_layer_forward(_ptr(X), B, S, h, heads, d, f, t, _ptr(ln1_g), _ptr(ln1_b), _shards(Wqkv),
                                  _ptr_array(bqkv), _shards(Wo), _ptr(bo), _ptr(ln2_g), _ptr(ln2_b), _shards(W1),
                                  _ptr_array(b1), _shards(W2), _ptr(b2), float(eps), 1 if causal else 0, _ptr(out),
                                  m, _ptr(ws), ws.numel(), _stream(stream)))
    return out


# ---------------------------------------------------------------- building blocks
def tp_layernorm_forward(x, gamma, beta, eps, y, stream=None):
    M, h = x.shape
    _check(lib().tp_layernorm_forward(_ptr(_dev(x)), _dtype_code(x), _ptr(gamma), _ptr(beta), M, h, float(eps),
                                      _ptr(_dev(y)), _dtype_code(y), _stream(stream)))
    return y


def tp_activation_forward(x, y, act="gelu", stream=None):
    """y = act(x) element-wise (fp32), as the column layer's epilogue applies it."""
    if x.dtype != torch.float32 or y.dtype != torch.float32:
        raise ValueError("fp32 tensors expected")
    _check(lib().tp_activation_forward(_ptr(_dev(x)), _ptr(_dev(y)), x.numel(), ACTS[act], _stream(stream)))
    return y


def tp_reduce_partials(P, bias, residual, out, stream=None):
    t, M, h = P.shape
    _check(lib().tp_reduce_partials(_ptr(_dev(P)), t, M, h, _ptr(bias), _ptr(residual), _dtype_code(out),
                                    _ptr(_dev(out)), _stream(stream)))
    return out


# ---------------------------------------------------------------- status and tracing
def tp_get_device_status(stream=None) -> int:
    return lib().tp_get_device_status(_stream(stream))


def tp_set_wait_limit_ns(ns: int):
    lib().tp_set_wait_limit_ns(int(ns))


def tp_selftest_bounded_wait(limit_ns: int, stream=None):
    _check(lib().tp_selftest_bounded_wait(int(limit_ns), _stream(stream)))


def tp_trace_enable(capacity: int = 4096):
    _check(lib().tp_trace_enable(capacity))


def tp_trace_disable():
    lib().tp_trace_disable()


def tp_trace_records():
    """[(kernel name, ms)] of the launches traced since tp_trace_enable (after a synchronise)."""
    out = []
    name = ctypes.c_char_p()
    ms = ctypes.c_float()
    for i in range(lib().tp_trace_count()):
        _check(lib().tp_trace_get(i, ctypes.byref(name), ctypes.byref(ms)))
        out.append((name.value.decode(), ms.value))
    return out
