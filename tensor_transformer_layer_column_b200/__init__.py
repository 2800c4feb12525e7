"""Python binding of libtplayer.so, the B200 tensor-parallel sublayer library.

Argument marshalling only: every entry point forwards device pointers and
sizes to the C ABI declared in include/tp_layer.h, and every step of the
computation runs in the library's CUDA kernels.  There is no CPU fallback:
if the shared library is missing, calling any entry point raises.

Tensors are ``torch`` CUDA tensors (bf16 unless stated) or raw integer
device addresses; ``None`` passes NULL.  The stream defaults to torch's
current stream of the tensors' device.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

__all__ = [
    "TpError", "Dims", "LayerParams", "LayerActs", "PostLNActs", "LayerGrads", "lib", "lib_path",
    "OP_MLP_FWD", "OP_MLP_BWD", "OP_ATTN_FWD", "OP_ATTN_BWD", "OP_LAYER_FWD", "OP_LAYER_BWD",
    "OP_POSTLN_FWD", "OP_POSTLN_BWD", "postln_layer_fwd", "postln_layer_bwd",
    "OP_LAYER_FWD_NOSAVE", "OP_LAYER_BWD_RECOMPUTE", "layer_fwd_nosave", "layer_bwd_recompute",
    "workspace_size", "check_error", "check_status", "version", "EXPORTED_SYMBOLS",
    "shard_cols", "unshard_cols", "shard_rows", "unshard_rows", "shard_qkv_heads",
    "unshard_qkv_heads", "mlp_fwd", "mlp_bwd", "attn_fwd", "attn_bwd", "layer_fwd", "layer_bwd",
    "layernorm_fwd", "layernorm_bwd", "layernorm_bwd_workspace_size", "layernorm_bwd_noalloc",
    "LaunchTrace", "GradReady", "layer_bwd_notify", "RANK_MLP_FWD", "RANK_MLP_BWD", "RANK_ATTN_FWD", "RANK_ATTN_BWD",
    "rank_workspace_size", "mlp_fwd_rank", "mlp_bwd_rank", "attn_fwd_rank", "attn_bwd_rank",
    "rowpar_finish", "layernorm_fwd_f16",
    "TRACE_KINDS", "selftest_wait_timeout",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_HERE, "libtplayer.so")

(OP_MLP_FWD, OP_MLP_BWD, OP_ATTN_FWD, OP_ATTN_BWD, OP_LAYER_FWD, OP_LAYER_BWD, OP_POSTLN_FWD,
 OP_POSTLN_BWD, OP_LAYER_FWD_NOSAVE, OP_LAYER_BWD_RECOMPUTE) = range(10)

RANK_MLP_FWD, RANK_MLP_BWD, RANK_ATTN_FWD, RANK_ATTN_BWD = range(4)

STATUS_NAMES = {0: "TP_OK", 1: "TP_ERR_INVALID_ARG", 2: "TP_ERR_UNSUPPORTED",
                3: "TP_ERR_MISALIGNED", 4: "TP_ERR_WORKSPACE", 5: "TP_ERR_CUDA",
                6: "TP_ERR_TIMEOUT", 7: "TP_ERR_RANGE"}


class TpError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")


class Dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("seq", ctypes.c_int), ("hidden", ctypes.c_int),
                ("ffn", ctypes.c_int), ("heads", ctypes.c_int), ("head_dim", ctypes.c_int),
                ("t", ctypes.c_int), ("causal", ctypes.c_int), ("ln_eps", ctypes.c_float)]

    @classmethod
    def of(cls, batch, seq, hidden, ffn=0, heads=0, head_dim=0, t=1, causal=1, ln_eps=1e-5):
        return cls(batch, seq, hidden, ffn, heads, head_dim, t, causal, ln_eps)


_P = ctypes.c_void_p


class LayerParams(ctypes.Structure):
    _fields_ = [(n, _P) for n in ("ln1_g", "ln1_b", "wqkv", "bqkv", "wout", "bout",
                                  "ln2_g", "ln2_b", "w1", "b1", "w2", "b2")]


class LayerActs(ctypes.Structure):
    _fields_ = [(n, _P) for n in ("u1", "mean1", "rstd1", "qkv", "o", "lse", "h", "u2",
                                  "mean2", "rstd2", "a", "hact", "wqkv16")]


class PostLNActs(ctypes.Structure):
    _fields_ = [(n, _P) for n in ("z1", "mean1", "rstd1", "qkv", "o", "lse", "h", "z2",
                                  "mean2", "rstd2", "a", "hact")]


class LayerGrads(ctypes.Structure):
    _fields_ = [(n, _P) for n in ("dln1_g", "dln1_b", "dwqkv", "dbqkv", "dwout", "dbout",
                                  "dln2_g", "dln2_b", "dw1", "db1", "dw2", "db2")]


class GradReady(ctypes.Structure):
    _fields_ = [(n, _P) for n in ("mlp", "attn", "ln1")]


# name -> argument types (all return tp_status unless listed in _RESTYPES)
_SIGS = {
    "tp_version": [],
    "tp_status_string": [ctypes.c_int],
    "tp_workspace_size": [ctypes.c_int, ctypes.POINTER(Dims)],
    "tp_check_error": [ctypes.POINTER(ctypes.c_uint)],
    "tp_shard_cols": [_P, ctypes.c_int, ctypes.c_int, ctypes.c_int, _P, _P],
    "tp_unshard_cols": [_P, ctypes.c_int, ctypes.c_int, ctypes.c_int, _P, _P],
    "tp_shard_rows": [_P, ctypes.c_int, ctypes.c_int, ctypes.c_int, _P, _P],
    "tp_unshard_rows": [_P, ctypes.c_int, ctypes.c_int, ctypes.c_int, _P, _P],
    "tp_shard_qkv_heads": [_P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, _P, _P],
    "tp_unshard_qkv_heads": [_P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, _P, _P],
    "tp_mlp_fwd": [ctypes.POINTER(Dims)] + [_P] * 9 + [_P, ctypes.c_size_t, _P],
    "tp_mlp_bwd": [ctypes.POINTER(Dims)] + [_P] * 12 + [_P, ctypes.c_size_t, _P],
    "tp_attn_fwd": [ctypes.POINTER(Dims)] + [_P] * 10 + [_P, ctypes.c_size_t, _P],
    "tp_attn_bwd": [ctypes.POINTER(Dims)] + [_P] * 13 + [_P, ctypes.c_size_t, _P],
    "tp_layer_fwd": [ctypes.POINTER(Dims), _P, ctypes.POINTER(LayerParams),
                     ctypes.POINTER(LayerActs), _P, _P, ctypes.c_size_t, _P],
    "tp_layer_bwd": [ctypes.POINTER(Dims), _P, ctypes.POINTER(LayerParams),
                     ctypes.POINTER(LayerActs), _P, _P, ctypes.POINTER(LayerGrads), _P,
                     ctypes.c_size_t, _P],
    "tp_layer_bwd_notify": [ctypes.POINTER(Dims), _P, ctypes.POINTER(LayerParams),
                            ctypes.POINTER(LayerActs), _P, _P, ctypes.POINTER(LayerGrads),
                            ctypes.POINTER(GradReady), _P, ctypes.c_size_t, _P],
    "tp_postln_layer_fwd": [ctypes.POINTER(Dims), _P, ctypes.POINTER(LayerParams),
                            ctypes.POINTER(PostLNActs), _P, _P, ctypes.c_size_t, _P],
    "tp_postln_layer_bwd": [ctypes.POINTER(Dims), _P, ctypes.POINTER(LayerParams),
                            ctypes.POINTER(PostLNActs), _P, _P, ctypes.POINTER(LayerGrads), _P,
                            ctypes.c_size_t, _P],
    "tp_layer_fwd_nosave": [ctypes.POINTER(Dims), _P, ctypes.POINTER(LayerParams), _P, _P,
                            ctypes.c_size_t, _P],
    "tp_layer_bwd_recompute": [ctypes.POINTER(Dims), _P, ctypes.POINTER(LayerParams), _P, _P,
                               ctypes.POINTER(LayerGrads), _P, ctypes.c_size_t, _P],
    "tp_layernorm_fwd": [_P, _P, _P, ctypes.c_int, ctypes.c_int, ctypes.c_float, _P, _P, _P, _P],
    "tp_layernorm_bwd_workspace_size": [ctypes.c_int, ctypes.c_int],
    "tp_layernorm_bwd": [_P, _P, _P, _P, _P, _P, ctypes.c_int, ctypes.c_int, _P, _P, _P, _P,
                         ctypes.c_size_t, _P],
    "tp_layernorm_bwd_noalloc": [_P, _P, _P, _P, _P, _P, ctypes.c_int, ctypes.c_int, _P, _P, _P,
                                 _P],
    "tp_selftest_wait_timeout": [ctypes.c_ulonglong, _P],
    "tp_rank_workspace_size": [ctypes.c_int, ctypes.POINTER(Dims)],
    "tp_mlp_fwd_rank": [ctypes.POINTER(Dims)] + [_P] * 7 + [_P],
    "tp_mlp_bwd_rank": [ctypes.POINTER(Dims)] + [_P] * 11 + [_P, ctypes.c_size_t, _P],
    "tp_attn_fwd_rank": [ctypes.POINTER(Dims)] + [_P] * 9 + [_P, ctypes.c_size_t, _P],
    "tp_attn_bwd_rank": [ctypes.POINTER(Dims)] + [_P] * 13 + [_P, ctypes.c_size_t, _P],
    "tp_rowpar_finish": [ctypes.POINTER(ctypes.c_void_p), ctypes.c_int, _P, _P, ctypes.c_int,
                         ctypes.c_int, _P, _P, _P],
    "tp_layernorm_fwd_f16": [_P, _P, _P, ctypes.c_int, ctypes.c_int, ctypes.c_float, _P, _P, _P,
                             _P],
    "tp_trace_begin": [ctypes.POINTER(ctypes.c_void_p), ctypes.POINTER(ctypes.c_int),
                       ctypes.POINTER(ctypes.c_double), ctypes.c_int],
    "tp_trace_end": [],
    "tp_attn_set_ds_limit": [ctypes.c_size_t],
}
_RESTYPES = {"tp_version": ctypes.c_char_p, "tp_status_string": ctypes.c_char_p,
             "tp_workspace_size": ctypes.c_size_t,
             "tp_layernorm_bwd_workspace_size": ctypes.c_size_t, "tp_trace_end": ctypes.c_int,
             "tp_rank_workspace_size": ctypes.c_size_t, "tp_attn_set_ds_limit": ctypes.c_size_t}
EXPORTED_SYMBOLS = tuple(_SIGS)

_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    """Load libtplayer.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(lib_path):
            raise RuntimeError(f"{lib_path} is missing: build it with "
                               "`python -m tensor_transformer_layer_column_b200.build`")
        handle = ctypes.CDLL(lib_path)
        for name, args in _SIGS.items():
            fn = getattr(handle, name)
            fn.argtypes = args
            fn.restype = _RESTYPES.get(name, ctypes.c_int)
        _lib = handle
    return _lib


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if not x.is_cuda:
        raise ValueError("tensor arguments must live on a CUDA device")
    if not x.is_contiguous():
        raise ValueError("tensor arguments must be contiguous")
    return x.data_ptr()


def _stream(stream, *tensors) -> Optional[int]:
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch
    for t in tensors:
        if t is not None and not isinstance(t, int):
            return torch.cuda.current_stream(t.device).cuda_stream
    return torch.cuda.current_stream().cuda_stream


def _check(status: int, where: str):
    if status != 0:
        raise TpError(status, where)


def version() -> str:
    return lib().tp_version().decode()


def workspace_size(op: int, dims: Dims) -> int:
    return lib().tp_workspace_size(op, ctypes.byref(dims))


def check_status():
    """Synchronise, read and clear the device error word: (status, code).

    status is 0 (TP_OK), 6 (TP_ERR_TIMEOUT: a bounded wait expired) or 7
    (TP_ERR_RANGE: a value stored as fp16 overflowed); code is the word."""
    code = ctypes.c_uint(0)
    st = lib().tp_check_error(ctypes.byref(code))
    if st not in (0, 6, 7):
        raise TpError(st, "tp_check_error")
    return st, code.value


def check_error() -> int:
    """Synchronise and return the device error word (0 if nothing was recorded)."""
    return check_status()[1]


def _ws(ws):
    if ws is None:
        return None, 0
    if isinstance(ws, tuple):
        return ws
    return ws.data_ptr(), ws.numel() * ws.element_size()


# ---------------------------------------------------------------- layout
def shard_cols(w, rows, cols, t, out, stream=None):
    _check(lib().tp_shard_cols(_ptr(w), rows, cols, t, _ptr(out), _stream(stream, w)), "tp_shard_cols")


def unshard_cols(p, rows, cols, t, out, stream=None):
    _check(lib().tp_unshard_cols(_ptr(p), rows, cols, t, _ptr(out), _stream(stream, p)), "tp_unshard_cols")


def shard_rows(w, rows, cols, t, out, stream=None):
    _check(lib().tp_shard_rows(_ptr(w), rows, cols, t, _ptr(out), _stream(stream, w)), "tp_shard_rows")


def unshard_rows(p, rows, cols, t, out, stream=None):
    _check(lib().tp_unshard_rows(_ptr(p), rows, cols, t, _ptr(out), _stream(stream, p)), "tp_unshard_rows")


def shard_qkv_heads(w, rows, hidden, heads, t, out, stream=None):
    _check(lib().tp_shard_qkv_heads(_ptr(w), rows, hidden, heads, t, _ptr(out), _stream(stream, w)),
           "tp_shard_qkv_heads")


def unshard_qkv_heads(p, rows, hidden, heads, t, out, stream=None):
    _check(lib().tp_unshard_qkv_heads(_ptr(p), rows, hidden, heads, t, _ptr(out),
                                      _stream(stream, p)), "tp_unshard_qkv_heads")


# ---------------------------------------------------------------- sublayers
def mlp_fwd(dims, x, w1, b1, w2, b2, resid, y, a_save, h_save, ws=None, stream=None):
    wp, wn = _ws(ws)
    _check(lib().tp_mlp_fwd(ctypes.byref(dims), _ptr(x), _ptr(w1), _ptr(b1), _ptr(w2), _ptr(b2),
                            _ptr(resid), _ptr(y), _ptr(a_save), _ptr(h_save), wp, wn,
                            _stream(stream, x)), "tp_mlp_fwd")


def mlp_bwd(dims, x, w1, w2, a_save, h_save, dy, dres, dx, dw1, dw2, db1, db2, ws, stream=None):
    wp, wn = _ws(ws)
    _check(lib().tp_mlp_bwd(ctypes.byref(dims), _ptr(x), _ptr(w1), _ptr(w2), _ptr(a_save),
                            _ptr(h_save), _ptr(dy), _ptr(dres), _ptr(dx), _ptr(dw1), _ptr(dw2),
                            _ptr(db1), _ptr(db2), wp, wn, _stream(stream, x)), "tp_mlp_bwd")


def attn_fwd(dims, x, wqkv, bqkv, wout, bout, resid, y, qkv_save, o_save, lse_save, ws=None,
             stream=None):
    wp, wn = _ws(ws)
    _check(lib().tp_attn_fwd(ctypes.byref(dims), _ptr(x), _ptr(wqkv), _ptr(bqkv), _ptr(wout),
                             _ptr(bout), _ptr(resid), _ptr(y), _ptr(qkv_save), _ptr(o_save),
                             _ptr(lse_save), wp, wn, _stream(stream, x)), "tp_attn_fwd")


def attn_bwd(dims, x, wqkv, wout, qkv_save, o_save, lse_save, dy, dres, dx, dwqkv, dbqkv, dwout,
             dbout, ws, stream=None):
    wp, wn = _ws(ws)
    _check(lib().tp_attn_bwd(ctypes.byref(dims), _ptr(x), _ptr(wqkv), _ptr(wout), _ptr(qkv_save),
                             _ptr(o_save), _ptr(lse_save), _ptr(dy), _ptr(dres), _ptr(dx),
                             _ptr(dwqkv), _ptr(dbqkv), _ptr(dwout), _ptr(dbout), wp, wn,
                             _stream(stream, x)), "tp_attn_bwd")


def _struct(cls, d):
    return cls(**{k: _ptr(v) for k, v in d.items()})


def layer_fwd(dims, x, params: dict, acts: dict, y, ws=None, stream=None):
    wp, wn = _ws(ws)
    p = _struct(LayerParams, params)
    a = _struct(LayerActs, acts)
    _check(lib().tp_layer_fwd(ctypes.byref(dims), _ptr(x), ctypes.byref(p), ctypes.byref(a),
                              _ptr(y), wp, wn, _stream(stream, x)), "tp_layer_fwd")


def layer_bwd(dims, x, params: dict, acts: dict, dy, dx, grads: dict, ws, stream=None):
    wp, wn = _ws(ws)
    p = _struct(LayerParams, params)
    a = _struct(LayerActs, acts)
    g = _struct(LayerGrads, grads)
    _check(lib().tp_layer_bwd(ctypes.byref(dims), _ptr(x), ctypes.byref(p), ctypes.byref(a),
                              _ptr(dy), _ptr(dx), ctypes.byref(g), wp, wn, _stream(stream, x)),
           "tp_layer_bwd")


def layer_bwd_notify(dims, x, params: dict, acts: dict, dy, dx, grads: dict, ready: dict, ws,
                     stream=None):
    """tp_layer_bwd that records ready["mlp"], ready["attn"], ready["ln1"]
    (torch.cuda.Event, already recorded once so that their handles exist) as
    each group of parameter gradients is enqueued."""
    wp, wn = _ws(ws)
    p = _struct(LayerParams, params)
    a = _struct(LayerActs, acts)
    g = _struct(LayerGrads, grads)
    r = GradReady(**{k: (None if ready.get(k) is None else ready[k].cuda_event)
                     for k in ("mlp", "attn", "ln1")})
    _check(lib().tp_layer_bwd_notify(ctypes.byref(dims), _ptr(x), ctypes.byref(p), ctypes.byref(a),
                                     _ptr(dy), _ptr(dx), ctypes.byref(g), ctypes.byref(r), wp, wn,
                                     _stream(stream, x)), "tp_layer_bwd_notify")


def postln_layer_fwd(dims, x, params: dict, acts: dict, y, ws=None, stream=None):
    wp, wn = _ws(ws)
    p = _struct(LayerParams, params)
    a = _struct(PostLNActs, acts)
    _check(lib().tp_postln_layer_fwd(ctypes.byref(dims), _ptr(x), ctypes.byref(p), ctypes.byref(a),
                                     _ptr(y), wp, wn, _stream(stream, x)), "tp_postln_layer_fwd")


def postln_layer_bwd(dims, x, params: dict, acts: dict, dy, dx, grads: dict, ws, stream=None):
    wp, wn = _ws(ws)
    p = _struct(LayerParams, params)
    a = _struct(PostLNActs, acts)
    g = _struct(LayerGrads, grads)
    _check(lib().tp_postln_layer_bwd(ctypes.byref(dims), _ptr(x), ctypes.byref(p), ctypes.byref(a),
                                     _ptr(dy), _ptr(dx), ctypes.byref(g), wp, wn,
                                     _stream(stream, x)), "tp_postln_layer_bwd")


def layer_fwd_nosave(dims, x, params: dict, y, ws, stream=None):
    wp, wn = _ws(ws)
    p = _struct(LayerParams, params)
    _check(lib().tp_layer_fwd_nosave(ctypes.byref(dims), _ptr(x), ctypes.byref(p), _ptr(y), wp, wn,
                                     _stream(stream, x)), "tp_layer_fwd_nosave")


def layer_bwd_recompute(dims, x, params: dict, dy, dx, grads: dict, ws, stream=None):
    wp, wn = _ws(ws)
    p = _struct(LayerParams, params)
    g = _struct(LayerGrads, grads)
    _check(lib().tp_layer_bwd_recompute(ctypes.byref(dims), _ptr(x), ctypes.byref(p), _ptr(dy),
                                        _ptr(dx), ctypes.byref(g), wp, wn, _stream(stream, x)),
           "tp_layer_bwd_recompute")


def attn_set_ds_limit(max_bytes: int) -> int:
    """Largest dS^T array (bytes) the attention backward keeps for its dq
    kernel (see include/tp_layer.h); returns the previous limit."""
    return int(lib().tp_attn_set_ds_limit(int(max_bytes)))


def selftest_wait_timeout(limit_ns: int, stream=None):
    """Enqueue the bounded-wait self-test (see include/tp_layer.h); read the
    outcome with check_error() afterwards."""
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    _check(lib().tp_selftest_wait_timeout(int(limit_ns), ctypes.c_void_p(s.cuda_stream)),
           "tp_selftest_wait_timeout")


def layernorm_fwd(x, gamma, beta, rows, D, eps, y, mean, rstd, stream=None):
    _check(lib().tp_layernorm_fwd(_ptr(x), _ptr(gamma), _ptr(beta), rows, D, eps, _ptr(y),
                                  _ptr(mean), _ptr(rstd), _stream(stream, x)), "tp_layernorm_fwd")


def layernorm_bwd_workspace_size(rows, D) -> int:
    return lib().tp_layernorm_bwd_workspace_size(rows, D)


def layernorm_bwd(dy, x, gamma, mean, rstd, dres, rows, D, dx, dgamma, dbeta, ws, stream=None):
    wp, wn = _ws(ws)
    _check(lib().tp_layernorm_bwd(_ptr(dy), _ptr(x), _ptr(gamma), _ptr(mean), _ptr(rstd),
                                  _ptr(dres), rows, D, _ptr(dx), _ptr(dgamma), _ptr(dbeta), wp,
                                  wn, _stream(stream, x)), "tp_layernorm_bwd")



def layernorm_bwd_noalloc(dy, x, gamma, mean, rstd, dres, rows, D, dx, dgamma, dbeta,
                          stream=None):
    """LayerNorm backward without a workspace (scratch is a static array in the library).

    For callers that cannot allocate device memory where they run the
    backward.  Calls on one device share the scratch: do not let two of them
    overlap on the GPU, and make the first call on a device outside stream
    capture.
    """
    _check(lib().tp_layernorm_bwd_noalloc(_ptr(dy), _ptr(x), _ptr(gamma), _ptr(mean), _ptr(rstd),
                                          _ptr(dres), rows, D, _ptr(dx), _ptr(dgamma),
                                          _ptr(dbeta), _stream(stream, x)),
           "tp_layernorm_bwd_noalloc")

# ---------------------------------------------------------------- one shard per GPU
def rank_workspace_size(op: int, dims: Dims) -> int:
    return lib().tp_rank_workspace_size(op, ctypes.byref(dims))


def mlp_fwd_rank(dims, x, w1_i, b1_i, w2_i, a_i, h_i, partial, stream=None):
    _check(lib().tp_mlp_fwd_rank(ctypes.byref(dims), _ptr(x), _ptr(w1_i), _ptr(b1_i), _ptr(w2_i),
                                 _ptr(a_i), _ptr(h_i), _ptr(partial), _stream(stream, x)),
           "tp_mlp_fwd_rank")


def mlp_bwd_rank(dims, x, w1_i, w2_i, a_i, h_i, dy, dw1_i, dw2_i, db1_i, db2, partial, ws,
                 stream=None):
    wp, wn = _ws(ws)
    _check(lib().tp_mlp_bwd_rank(ctypes.byref(dims), _ptr(x), _ptr(w1_i), _ptr(w2_i), _ptr(a_i),
                                 _ptr(h_i), _ptr(dy), _ptr(dw1_i), _ptr(dw2_i), _ptr(db1_i),
                                 _ptr(db2), _ptr(partial), wp, wn, _stream(stream, dy)),
           "tp_mlp_bwd_rank")


def attn_fwd_rank(dims, x, x16, wqkv_i, bqkv_i, wout_i, qkv_i, o_i, lse_i, partial, ws,
                  stream=None):
    wp, wn = _ws(ws)
    _check(lib().tp_attn_fwd_rank(ctypes.byref(dims), _ptr(x), _ptr(x16), _ptr(wqkv_i),
                                  _ptr(bqkv_i), _ptr(wout_i), _ptr(qkv_i), _ptr(o_i), _ptr(lse_i),
                                  _ptr(partial), wp, wn, _stream(stream, wqkv_i)),
           "tp_attn_fwd_rank")


def attn_bwd_rank(dims, x, x16, wqkv_i, wout_i, qkv_i, o_i, lse_i, dy, dwqkv_i, dbqkv_i, dwout_i,
                  dbout, partial, ws, stream=None):
    wp, wn = _ws(ws)
    _check(lib().tp_attn_bwd_rank(ctypes.byref(dims), _ptr(x), _ptr(x16), _ptr(wqkv_i),
                                  _ptr(wout_i), _ptr(qkv_i), _ptr(o_i), _ptr(lse_i), _ptr(dy),
                                  _ptr(dwqkv_i), _ptr(dbqkv_i), _ptr(dwout_i), _ptr(dbout),
                                  _ptr(partial), wp, wn, _stream(stream, dy)),
           "tp_attn_bwd_rank")


def rowpar_finish(parts, bias, resid, rows, cols, out, out32=None, stream=None):
    """out = bf16(sum of the fp32 buffers in `parts`, in order, + bias + resid)."""
    arr = (ctypes.c_void_p * len(parts))(*[_ptr(q) for q in parts])
    _check(lib().tp_rowpar_finish(arr, len(parts), _ptr(bias), _ptr(resid), rows, cols, _ptr(out),
                                  _ptr(out32), _stream(stream, out)), "tp_rowpar_finish")


def layernorm_fwd_f16(x, gamma, beta, rows, D, eps, y, mean, rstd, stream=None):
    _check(lib().tp_layernorm_fwd_f16(_ptr(x), _ptr(gamma), _ptr(beta), rows, D, eps, _ptr(y),
                                      _ptr(mean), _ptr(rstd), _stream(stream, x)),
           "tp_layernorm_fwd_f16")


TRACE_KINDS = ("gemm", "attn_fwd", "attn_bwd_prep", "attn_bwd_dkdv", "attn_bwd_dq", "ln_fwd",
               "ln_bwd", "ln_param", "colsum", "layout", "cast", "finish")


class LaunchTrace:
    """Context manager around tp_trace_begin / tp_trace_end.

    Inside the block every kernel the library enqueues is bracketed by CUDA
    events on its own stream; afterwards ``records()`` gives, per launch, its
    class name, algorithmic FLOPs and device duration in milliseconds.
    """

    def __init__(self, capacity: int):
        import torch
        self.capacity = capacity
        self._events = [torch.cuda.Event(enable_timing=True) for _ in range(2 * capacity)]
        for e in self._events:       # materialise the underlying cudaEvent_t handles
            e.record()
        torch.cuda.synchronize()
        self._handles = (ctypes.c_void_p * (2 * capacity))(*[e.cuda_event for e in self._events])
        self._kinds = (ctypes.c_int * capacity)()
        self._flops = (ctypes.c_double * capacity)()
        self.count = 0

    def __enter__(self):
        _check(lib().tp_trace_begin(self._handles, self._kinds, self._flops, self.capacity),
               "tp_trace_begin")
        return self

    def __exit__(self, *exc):
        self.count = lib().tp_trace_end()
        return False

    def records(self):
        import torch
        torch.cuda.synchronize()
        n = min(self.count, self.capacity)
        out = []
        for i in range(n):
            ms = self._events[2 * i].elapsed_time(self._events[2 * i + 1])
            out.append((TRACE_KINDS[self._kinds[i]], float(self._flops[i]), ms))
        return out
