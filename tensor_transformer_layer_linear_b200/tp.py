"""Thin ctypes binding of libtp.so (the C ABI declared in include/tp.h).

Argument marshalling only: tensors are passed as raw device pointers
(``data_ptr()``), the stream as the raw ``cudaStream_t`` of torch's current
stream unless one is given. Every step of the computation runs in the
library's CUDA kernels; there is no CPU or PyTorch fallback, and importing
this module fails loudly if the library has not been built.

Function names are those of the C ABI. bf16 tensors may be given as
``torch.bfloat16`` or ``torch.int16`` (bit patterns); fp32 partials as
``torch.float32``. All tensors must be contiguous CUDA tensors.
"""
from __future__ import annotations

import ctypes
import os
import re

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libtp.so")
HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "tp.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with "
        "`python -m tensor_transformer_layer_linear_b200.build` (nvcc, sm_100a)")

lib = ctypes.CDLL(LIB_PATH)

# status codes and enums (include/tp.h)
TP_OK, TP_ERR_NULL, TP_ERR_SHAPE, TP_ERR_ALIGN = 0, 1, 2, 3
TP_ERR_WORKSPACE, TP_ERR_UNSUPPORTED, TP_ERR_CUDA, TP_ERR_TIMEOUT = 4, 5, 6, 7
TP_SPLIT_COLUMN, TP_SPLIT_ROW, TP_SPLIT_QKV_HEADS, TP_SPLIT_GATE_UP = 0, 1, 2, 3
TP_ACT_NONE, TP_ACT_GELU_ERF, TP_ACT_SWIGLU = 0, 1, 2
TP_WS_MLP, TP_WS_ATTN, TP_WS_LAYER, TP_WS_LAYER_SP, TP_WS_MLP_BWD = 0, 1, 2, 3, 4
TP_WS_ATTN_CORE_BWD, TP_WS_ATTN_BWD, TP_WS_LAYER_BWD, TP_WS_LN_BWD, TP_WS_LAYER_BWD_SP = 5, 6, 7, 8, 9

_vp, _i64, _i32, _f32, _sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_size_t


class tp_layer_weights(ctypes.Structure):
    _fields_ = [(n, _vp) for n in (
        "ln1_gamma", "ln1_beta", "Wqkv_shards", "bqkv_shards", "Wo_shards", "bo",
        "ln2_gamma", "ln2_beta", "A_shards", "b1_shards", "B_shards", "b2")]


class tp_layer_grads(ctypes.Structure):
    _fields_ = [(n, _vp) for n in (
        "ln1_gamma", "ln1_beta", "Wqkv_shards", "bqkv_shards", "Wo_shards", "bo",
        "ln2_gamma", "ln2_beta", "A_shards", "b1_shards", "B_shards", "b2")]


_SIGS = {
    "tp_shard_weights": (_i32, [_vp, _i64, _i64, _i32, _i32, _i64, _vp, _vp]),
    "tp_shard_index_map": (_i32, [_i32, _i64, _i64, _i32, _i64, _vp, _vp]),
    "tp_column_linear": (_i32, [_vp, _i64, _i64, _vp, _vp, _i64, _i32, _i32, _vp, _vp]),
    "tp_row_linear": (_i32, [_vp, _i64, _i64, _vp, _i64, _i32, _vp, _vp]),
    "tp_reduce_partials": (_i32, [_vp, _i32, _i64, _i64, _vp, _vp, _vp, _vp]),
    "tp_reduce_partials_layernorm": (_i32, [_vp, _i32, _i64, _i64, _vp, _vp, _vp, _vp, _f32,
                                            _vp, _vp, _vp]),
    "tp_layernorm": (_i32, [_vp, _i64, _i64, _vp, _vp, _f32, _vp, _vp]),
    "tp_attention": (_i32, [_vp, _i64, _i64, _i64, _i64, _i32, _i32, _vp, _vp]),
    "tp_mlp_forward": (_i32, [_vp, _i64, _i64, _i64, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _sz,
                              _vp, _vp]),
    "tp_attn_forward": (_i32, [_vp, _i64, _i64, _i64, _i64, _i32, _i32, _vp, _vp, _vp, _vp, _vp,
                               _vp, _sz, _vp, _vp]),
    "tp_layer_forward": (_i32, [_vp, _i64, _i64, _i64, _i64, _i64, _i32,
                                ctypes.POINTER(tp_layer_weights), _f32, _vp, _sz, _vp, _vp]),
    "tp_mlp_forward_swiglu": (_i32, [_vp, _i64, _i64, _i64, _i32, _vp, _vp, _vp, _vp, _vp, _sz,
                                     _vp, _vp]),
    "tp_mlp_forward_noalloc": (_i32, [_vp, _i64, _i64, _i64, _i32, _vp, _vp, _vp, _vp, _vp, _vp,
                                      _vp]),
    "tp_reduce_scatter_partials": (_i32, [_vp, _i32, _i64, _i64, _i64, _vp, _vp, _vp, _vp]),
    "tp_all_gather_sequence": (_i32, [_vp, _i32, _i64, _i64, _i64, _vp, _vp]),
    "tp_layer_forward_sp": (_i32, [_vp, _i64, _i64, _i64, _i64, _i64, _i32,
                                   ctypes.POINTER(tp_layer_weights), _f32, _vp, _sz, _vp, _vp]),
    "tp_shard_qkv_gqa": (_i32, [_vp, _i64, _i64, _i64, _i64, _i32, _vp, _vp]),
    "tp_attention_gqa": (_i32, [_vp, _i64, _i64, _i64, _i64, _i64, _i32, _i32, _vp, _vp]),
    "tp_attn_forward_gqa": (_i32, [_vp, _i64, _i64, _i64, _i64, _i64, _i32, _i32, _vp, _vp, _vp,
                                   _vp, _vp, _vp, _sz, _vp, _vp]),
    "tp_mlp_backward": (_i32, [_vp, _i64, _i64, _i64, _i32, _vp, _vp, _vp, _vp, _i32, _vp, _sz,
                               _vp, _vp, _vp, _vp, _vp, _vp]),
    "tp_attention_lse": (_i32, [_vp, _i64, _i64, _i64, _i64, _i32, _i32, _vp, _vp, _vp]),
    "tp_attention_backward": (_i32, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _i32, _i32,
                                     _vp, _sz, _vp, _vp]),
    "tp_attn_backward": (_i32, [_vp, _i64, _i64, _i64, _i64, _i32, _i32, _vp, _vp, _vp, _vp,
                                _i32, _vp, _sz, _vp, _vp, _vp, _vp, _vp, _vp]),
    "tp_reduce_partials_layernorm_backward": (_i32, [_vp, _i32, _i64, _i64, _vp, _vp, _vp, _f32,
                                                     _vp, _sz, _vp, _vp, _vp, _vp]),
    "tp_layer_backward": (_i32, [_vp, _i64, _i64, _i64, _i64, _i64, _i32,
                                 ctypes.POINTER(tp_layer_weights), _f32, _vp, _vp, _sz, _vp,
                                 ctypes.POINTER(tp_layer_grads), _vp]),
    "tp_attention_gqa_lse": (_i32, [_vp, _i64, _i64, _i64, _i64, _i64, _i32, _i32, _vp, _vp,
                                    _vp]),
    "tp_attention_gqa_backward": (_i32, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64, _i32,
                                         _i32, _vp, _sz, _vp, _vp]),
    "tp_attn_backward_gqa": (_i32, [_vp, _i64, _i64, _i64, _i64, _i64, _i32, _i32, _vp, _vp, _vp,
                                    _vp, _i32, _vp, _sz, _vp, _vp, _vp, _vp, _vp, _vp]),
    "tp_layer_backward_sp": (_i32, [_vp, _i64, _i64, _i64, _i64, _i64, _i32,
                                    ctypes.POINTER(tp_layer_weights), _f32, _vp, _vp, _sz, _vp,
                                    ctypes.POINTER(tp_layer_grads), _vp]),
    "tp_workspace_bytes": (_sz, [_i32, _i64, _i64, _i64, _i32]),
    "tp_get_last_error": (_i32, [_vp]),
    "tp_selftest_wait_timeout": (_i32, [_i64, _vp]),
    "tp_status_string": (ctypes.c_char_p, [_i32]),
    "tp_trace_begin": (_i32, [_i32]),
    "tp_trace_end": (_i32, []),
    "tp_trace_record": (_i32, [_i32, ctypes.POINTER(_i32), ctypes.POINTER(_f32)]),
    "tp_kernel_name": (ctypes.c_char_p, [_i32]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


def header_functions() -> list:
    """Names of every function include/tp.h declares."""
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(tp_[a-z_0-9]+)\s*\(",
                                 text, flags=re.M)))


class TPError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {lib.tp_status_string(status).decode()}")


def _check(st: int, where: str) -> None:
    if st != TP_OK:
        raise TPError(st, where)


def _p(t) -> int:
    """Raw pointer of a tensor (None -> NULL; ints pass through)."""
    if t is None:
        return 0
    if isinstance(t, int):
        return t
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    if t.device.type != "cuda":
        raise ValueError("tensor must be on a CUDA device")
    return t.data_ptr()


def _s(stream) -> int:
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch
    return torch.cuda.current_stream().cuda_stream


def tp_status_string(status: int) -> str:
    return lib.tp_status_string(status).decode()


def tp_workspace_bytes(kind: int, tokens: int, h: int, ffn: int, n_shards: int) -> int:
    return int(lib.tp_workspace_bytes(kind, tokens, h, ffn, n_shards))


def tp_shard_index_map(kind: int, h_in: int, h_out: int, n_shards: int, head_dim: int = 0):
    """Host-only index map -> (owner int32 array, local int64 array)."""
    import numpy as np
    n = h_in if kind == TP_SPLIT_ROW else h_out
    owner = np.zeros(n, dtype=np.int32)
    local = np.zeros(n, dtype=np.int64)
    _check(lib.tp_shard_index_map(kind, h_in, h_out, n_shards, head_dim,
                                  owner.ctypes.data, local.ctypes.data), "tp_shard_index_map")
    return owner, local


def tp_shard_weights(W, h_in, h_out, n_shards, kind, head_dim, W_shards, stream=None):
    _check(lib.tp_shard_weights(_p(W), h_in, h_out, n_shards, kind, head_dim, _p(W_shards),
                                _s(stream)), "tp_shard_weights")


def tp_column_linear(X, B, h_in, W_shards, bias_shards, h_out, n_shards, act, Y_shards,
                     stream=None):
    _check(lib.tp_column_linear(_p(X), B, h_in, _p(W_shards), _p(bias_shards), h_out, n_shards,
                                act, _p(Y_shards), _s(stream)), "tp_column_linear")


def tp_row_linear(X_shards, B, h_in, W_shards, h_out, n_shards, partials, stream=None):
    _check(lib.tp_row_linear(_p(X_shards), B, h_in, _p(W_shards), h_out, n_shards, _p(partials),
                             _s(stream)), "tp_row_linear")


def tp_reduce_partials(partials, n_shards, B, h_out, bias, residual, Y, stream=None):
    _check(lib.tp_reduce_partials(_p(partials), n_shards, B, h_out, _p(bias), _p(residual), _p(Y),
                                  _s(stream)), "tp_reduce_partials")


def tp_reduce_partials_layernorm(partials, n_shards, B, h_out, bias, residual, gamma, beta, eps,
                                 Y_sum, Y_ln, stream=None):
    _check(lib.tp_reduce_partials_layernorm(_p(partials), n_shards, B, h_out, _p(bias),
                                            _p(residual), _p(gamma), _p(beta), eps, _p(Y_sum),
                                            _p(Y_ln), _s(stream)),
           "tp_reduce_partials_layernorm")


def tp_layernorm(X, B, h, gamma, beta, eps, Y, stream=None):
    _check(lib.tp_layernorm(_p(X), B, h, _p(gamma), _p(beta), eps, _p(Y), _s(stream)),
           "tp_layernorm")


def tp_attention(QKV_shards, batch, seq, h, n_heads, causal, n_shards, O_shards, stream=None):
    _check(lib.tp_attention(_p(QKV_shards), batch, seq, h, n_heads, int(bool(causal)), n_shards,
                            _p(O_shards), _s(stream)), "tp_attention")


def tp_mlp_forward(X, B, h, ffn, n_shards, A_shards, b1_shards, B_shards, b2, residual, ws,
                   ws_bytes, Y, stream=None):
    _check(lib.tp_mlp_forward(_p(X), B, h, ffn, n_shards, _p(A_shards), _p(b1_shards),
                              _p(B_shards), _p(b2), _p(residual), _p(ws), ws_bytes, _p(Y),
                              _s(stream)), "tp_mlp_forward")


def tp_mlp_forward_swiglu(X, B, h, ffn, n_shards, GU_shards, B_shards, b2, residual, ws,
                          ws_bytes, Y, stream=None):
    _check(lib.tp_mlp_forward_swiglu(_p(X), B, h, ffn, n_shards, _p(GU_shards), _p(B_shards),
                                     _p(b2), _p(residual), _p(ws), ws_bytes, _p(Y), _s(stream)),
           "tp_mlp_forward_swiglu")


TP_NOALLOC_WS_BYTES = 32 * 1024 * 1024


def tp_mlp_forward_noalloc(X, B, h, ffn, n_shards, A_shards, b1_shards, B_shards, b2, residual,
                           Y, stream=None):
    """tp_mlp_forward without a workspace argument, for callers that cannot
    allocate device memory: the intermediates live in the library's fixed
    TP_NOALLOC_WS_BYTES device array (shared by all calls on a device; calls
    that overlap on the GPU race on it)."""
    _check(lib.tp_mlp_forward_noalloc(_p(X), B, h, ffn, n_shards, _p(A_shards), _p(b1_shards),
                                      _p(B_shards), _p(b2), _p(residual), _p(Y), _s(stream)),
           "tp_mlp_forward_noalloc")


def tp_attn_forward(X, batch, seq, h, n_heads, causal, n_shards, Wqkv_shards, bqkv_shards,
                    Wo_shards, bo, residual, ws, ws_bytes, Y, stream=None):
    _check(lib.tp_attn_forward(_p(X), batch, seq, h, n_heads, int(bool(causal)), n_shards,
                               _p(Wqkv_shards), _p(bqkv_shards), _p(Wo_shards), _p(bo),
                               _p(residual), _p(ws), ws_bytes, _p(Y), _s(stream)),
           "tp_attn_forward")


def make_layer_weights(**tensors) -> tp_layer_weights:
    """Build the tp_layer_weights struct from tensors named like its fields.

    The struct holds raw device addresses, so it also keeps a reference to
    every tensor it was built from: the memory stays allocated for as long as
    the struct lives, even when the caller passed temporaries (otherwise
    torch's caching allocator could hand those bytes to the next tensor, e.g.
    the workspace, and the layer would read its own scratch as weights)."""
    w = tp_layer_weights()
    for name, _ in tp_layer_weights._fields_:
        setattr(w, name, _p(tensors.get(name)))
    w._tensors = dict(tensors)
    return w


def tp_layer_forward(X, batch, seq, h, n_heads, ffn, n_shards, weights: tp_layer_weights,
                     ln_eps, ws, ws_bytes, Y, stream=None):
    _check(lib.tp_layer_forward(_p(X), batch, seq, h, n_heads, ffn, n_shards,
                                ctypes.byref(weights), ln_eps, _p(ws), ws_bytes, _p(Y),
                                _s(stream)), "tp_layer_forward")


def tp_reduce_scatter_partials(partials, n_shards, batch, seq, h, bias, residual_shards,
                               Y_shards, stream=None):
    _check(lib.tp_reduce_scatter_partials(_p(partials), n_shards, batch, seq, h, _p(bias),
                                          _p(residual_shards), _p(Y_shards), _s(stream)),
           "tp_reduce_scatter_partials")


def tp_all_gather_sequence(X_shards, n_shards, batch, seq, h, X, stream=None):
    _check(lib.tp_all_gather_sequence(_p(X_shards), n_shards, batch, seq, h, _p(X), _s(stream)),
           "tp_all_gather_sequence")


def tp_layer_forward_sp(X_shards, batch, seq, h, n_heads, ffn, n_shards,
                        weights: tp_layer_weights, ln_eps, ws, ws_bytes, Y_shards, stream=None):
    _check(lib.tp_layer_forward_sp(_p(X_shards), batch, seq, h, n_heads, ffn, n_shards,
                                   ctypes.byref(weights), ln_eps, _p(ws), ws_bytes, _p(Y_shards),
                                   _s(stream)), "tp_layer_forward_sp")


def tp_shard_qkv_gqa(W, h_in, n_q, n_kv, head_dim, n_shards, W_shards, stream=None):
    _check(lib.tp_shard_qkv_gqa(_p(W), h_in, n_q, n_kv, head_dim, n_shards, _p(W_shards),
                                _s(stream)), "tp_shard_qkv_gqa")


def tp_attention_gqa(QKV_shards, batch, seq, n_q, n_kv, head_dim, causal, n_shards, O_shards,
                     stream=None):
    _check(lib.tp_attention_gqa(_p(QKV_shards), batch, seq, n_q, n_kv, head_dim,
                                int(bool(causal)), n_shards, _p(O_shards), _s(stream)),
           "tp_attention_gqa")


def tp_attn_forward_gqa(X, batch, seq, h, n_q, n_kv, causal, n_shards, Wqkv_shards, bqkv_shards,
                        Wo_shards, bo, residual, ws, ws_bytes, Y, stream=None):
    _check(lib.tp_attn_forward_gqa(_p(X), batch, seq, h, n_q, n_kv, int(bool(causal)), n_shards,
                                   _p(Wqkv_shards), _p(bqkv_shards), _p(Wo_shards), _p(bo),
                                   _p(residual), _p(ws), ws_bytes, _p(Y), _s(stream)),
           "tp_attn_forward_gqa")


def tp_mlp_backward(X, B, h, ffn, n_shards, A_shards, b1_shards, B_shards, dY, residual, ws,
                    ws_bytes, dX, dA_shards, db1, dB_shards, db2, stream=None):
    _check(lib.tp_mlp_backward(_p(X), B, h, ffn, n_shards, _p(A_shards), _p(b1_shards),
                               _p(B_shards), _p(dY), int(bool(residual)), _p(ws), ws_bytes, _p(dX),
                               _p(dA_shards), _p(db1), _p(dB_shards), _p(db2), _s(stream)),
           "tp_mlp_backward")


def tp_attention_lse(QKV_shards, batch, seq, h, n_heads, causal, n_shards, O_shards, lse,
                     stream=None):
    _check(lib.tp_attention_lse(_p(QKV_shards), batch, seq, h, n_heads, int(bool(causal)),
                                n_shards, _p(O_shards), _p(lse), _s(stream)), "tp_attention_lse")


def tp_attention_backward(QKV_shards, O_shards, dO_shards, lse, batch, seq, h, n_heads, causal,
                          n_shards, ws, ws_bytes, dQKV_shards, stream=None):
    _check(lib.tp_attention_backward(_p(QKV_shards), _p(O_shards), _p(dO_shards), _p(lse), batch,
                                     seq, h, n_heads, int(bool(causal)), n_shards, _p(ws),
                                     ws_bytes, _p(dQKV_shards), _s(stream)),
           "tp_attention_backward")


def tp_attn_backward(X, batch, seq, h, n_heads, causal, n_shards, Wqkv_shards, bqkv_shards,
                     Wo_shards, dY, residual, ws, ws_bytes, dX, dWqkv_shards, dbqkv_shards,
                     dWo_shards, dbo, stream=None):
    _check(lib.tp_attn_backward(_p(X), batch, seq, h, n_heads, int(bool(causal)), n_shards,
                                _p(Wqkv_shards), _p(bqkv_shards), _p(Wo_shards), _p(dY),
                                int(bool(residual)), _p(ws), ws_bytes, _p(dX), _p(dWqkv_shards),
                                _p(dbqkv_shards), _p(dWo_shards), _p(dbo), _s(stream)),
           "tp_attn_backward")


def tp_reduce_partials_layernorm_backward(partials, n_shards, B, h, x, gamma, residual_grad, eps,
                                          ws, ws_bytes, dX, dgamma, dbeta, stream=None):
    _check(lib.tp_reduce_partials_layernorm_backward(
        _p(partials), n_shards, B, h, _p(x), _p(gamma), _p(residual_grad), eps, _p(ws), ws_bytes,
        _p(dX), _p(dgamma), _p(dbeta), _s(stream)), "tp_reduce_partials_layernorm_backward")


def make_layer_grads(**tensors) -> tp_layer_grads:
    """Build the tp_layer_grads struct from fp32 tensors named like its fields
    (the struct keeps a reference to each, as make_layer_weights does)."""
    g = tp_layer_grads()
    for name, _ in tp_layer_grads._fields_:
        setattr(g, name, _p(tensors.get(name)))
    g._tensors = dict(tensors)
    return g


def tp_layer_backward(X, batch, seq, h, n_heads, ffn, n_shards, weights: tp_layer_weights, ln_eps,
                      dY, ws, ws_bytes, dX, grads: tp_layer_grads, stream=None):
    _check(lib.tp_layer_backward(_p(X), batch, seq, h, n_heads, ffn, n_shards,
                                 ctypes.byref(weights), ln_eps, _p(dY), _p(ws), ws_bytes, _p(dX),
                                 ctypes.byref(grads), _s(stream)), "tp_layer_backward")


def tp_attention_gqa_lse(QKV_shards, batch, seq, n_q, n_kv, head_dim, causal, n_shards, O_shards,
                         lse, stream=None):
    _check(lib.tp_attention_gqa_lse(_p(QKV_shards), batch, seq, n_q, n_kv, head_dim,
                                    int(bool(causal)), n_shards, _p(O_shards), _p(lse), _s(stream)),
           "tp_attention_gqa_lse")


def tp_attention_gqa_backward(QKV_shards, O_shards, dO_shards, lse, batch, seq, n_q, n_kv,
                              head_dim, causal, n_shards, ws, ws_bytes, dQKV_shards, stream=None):
    _check(lib.tp_attention_gqa_backward(_p(QKV_shards), _p(O_shards), _p(dO_shards), _p(lse),
                                         batch, seq, n_q, n_kv, head_dim, int(bool(causal)),
                                         n_shards, _p(ws), ws_bytes, _p(dQKV_shards), _s(stream)),
           "tp_attention_gqa_backward")


def tp_attn_backward_gqa(X, batch, seq, h, n_q, n_kv, causal, n_shards, Wqkv_shards, bqkv_shards,
                         Wo_shards, dY, residual, ws, ws_bytes, dX, dWqkv_shards, dbqkv_shards,
                         dWo_shards, dbo, stream=None):
    _check(lib.tp_attn_backward_gqa(_p(X), batch, seq, h, n_q, n_kv, int(bool(causal)), n_shards,
                                    _p(Wqkv_shards), _p(bqkv_shards), _p(Wo_shards), _p(dY),
                                    int(bool(residual)), _p(ws), ws_bytes, _p(dX),
                                    _p(dWqkv_shards), _p(dbqkv_shards), _p(dWo_shards), _p(dbo),
                                    _s(stream)), "tp_attn_backward_gqa")


def tp_layer_backward_sp(X_shards, batch, seq, h, n_heads, ffn, n_shards,
                         weights: tp_layer_weights, ln_eps, dY_shards, ws, ws_bytes, dX_shards,
                         grads: tp_layer_grads, stream=None):
    _check(lib.tp_layer_backward_sp(_p(X_shards), batch, seq, h, n_heads, ffn, n_shards,
                                    ctypes.byref(weights), ln_eps, _p(dY_shards), _p(ws), ws_bytes,
                                    _p(dX_shards), ctypes.byref(grads), _s(stream)),
           "tp_layer_backward_sp")


def tp_get_last_error(stream=None) -> int:
    return int(lib.tp_get_last_error(_s(stream)))


def tp_selftest_wait_timeout(limit_us, stream=None):
    _check(lib.tp_selftest_wait_timeout(limit_us, _s(stream)), "tp_selftest_wait_timeout")


def tp_trace_begin(max_records: int) -> None:
    _check(lib.tp_trace_begin(max_records), "tp_trace_begin")


def tp_trace_end() -> list:
    """Stop the trace; return [(kernel_name, ms), ...] for the timed launches
    and, as a second value, the number of launches seen."""
    seen = lib.tp_trace_end()
    recs = []
    k = 0
    while True:
        kid, ms = _i32(), _f32()
        if lib.tp_trace_record(k, ctypes.byref(kid), ctypes.byref(ms)) != TP_OK:
            break
        recs.append((lib.tp_kernel_name(kid.value).decode(), float(ms.value)))
        k += 1
    return recs, int(seen)
