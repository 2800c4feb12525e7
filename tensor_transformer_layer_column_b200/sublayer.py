"""torch-facing wrappers of the C ABI: the sharded MLP, attention and pre-LN layer.

Each object takes UNSHARDED bf16 CUDA weights (the orientation of
``output = GeLU(x W1) W2``: weights are [in, out]), packs them into the
shard layouts with the library's own layout kernels, and owns the device
buffers of one forward/backward pass.  torch is used for allocation and
streams only; all arithmetic happens in libtplayer.so.
"""
from __future__ import annotations

import functools
from typing import Dict, Optional

import torch

from . import (Dims, OP_ATTN_BWD, OP_ATTN_FWD, OP_LAYER_BWD, OP_LAYER_BWD_RECOMPUTE,
               OP_LAYER_FWD, OP_LAYER_FWD_NOSAVE, OP_MLP_BWD, OP_POSTLN_BWD, OP_POSTLN_FWD,
               attn_bwd, attn_fwd, layer_bwd, layer_bwd_notify, layer_bwd_recompute, layer_fwd,
               layer_fwd_nosave,
               mlp_bwd, mlp_fwd, postln_layer_bwd, postln_layer_fwd, shard_cols,
               shard_qkv_heads, shard_rows, unshard_cols, unshard_qkv_heads, workspace_size)

BF16 = torch.bfloat16


def _empty(shape, dtype=BF16, device="cuda"):
    return torch.empty(shape, dtype=dtype, device=device)


def _expect(name, t, shape, dtype=BF16, device=None, optional=False):
    """Check a tensor argument before any library call: the C ABI takes raw
    pointers, so a wrong shape or dtype would otherwise be read as garbage or
    past the end of the buffer."""
    if t is None:
        if optional:
            return
        raise ValueError(f"{name} is required")
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if device is not None and t.device != torch.device(device):
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def _expect_all(given: Dict, spec: Dict, device, what: str, optional=()):
    """Every tensor of a caller-provided buffer dict against its (shape, dtype);
    keys in `optional` may be absent or None."""
    for k, (shape, dtype) in spec.items():
        _expect(f"{what}[{k!r}]", given.get(k), shape, dtype, device, optional=k in optional)


def pack_cols(w: torch.Tensor, t: int) -> torch.Tensor:
    rows, cols = w.shape
    out = _empty((t, rows, cols // t), device=w.device)
    shard_cols(w, rows, cols, t, out)
    return out


def unpack_cols(p: torch.Tensor) -> torch.Tensor:
    t, rows, ct = p.shape
    out = _empty((rows, t * ct), device=p.device)
    unshard_cols(p, rows, t * ct, t, out)
    return out


def pack_rows(w: torch.Tensor, t: int) -> torch.Tensor:
    rows, cols = w.shape
    out = _empty((t, rows // t, cols), device=w.device)
    shard_rows(w, rows, cols, t, out)
    return out


def pack_qkv(w: torch.Tensor, heads: int, t: int) -> torch.Tensor:
    """[rows, 3D] (or a [3D] bias) -> [t][rows][3D/t]."""
    w2 = w.reshape(-1, w.shape[-1])
    rows, c3 = w2.shape
    out = _empty((t, rows, c3 // t), device=w.device)
    shard_qkv_heads(w2, rows, c3 // 3, heads, t, out)
    return out


def unpack_qkv(p: torch.Tensor, heads: int) -> torch.Tensor:
    t, rows, c3t = p.shape
    out = _empty((rows, c3t * t), device=p.device)
    unshard_qkv_heads(p, rows, c3t * t // 3, heads, t, out)
    return out


def _nvtx(name: str):
    """Wrap a sublayer call in an NVTX range (for timeline profilers)."""
    def deco(fn):
        @functools.wraps(fn)
        def wrapper(*args, **kwargs):
            torch.cuda.nvtx.range_push(name)
            try:
                return fn(*args, **kwargs)
            finally:
                torch.cuda.nvtx.range_pop()
        return wrapper
    return deco


def _ws(op: int, dims: Dims, device) -> Optional[torch.Tensor]:
    n = workspace_size(op, dims)
    return torch.empty(max(n, 1), dtype=torch.uint8, device=device) if n else None


class ShardedMLP:
    """Column-parallel W1 + local GeLU, row-parallel W2 + shard sum, on one GPU."""

    def __init__(self, dims: Dims, w1, b1, w2, b2):
        self.dims = dims
        t = dims.t
        D, F = dims.hidden, dims.ffn
        dev = w1.device if isinstance(w1, torch.Tensor) else None
        _expect("w1", w1, (D, F), device=dev)
        _expect("b1", b1, (F,), device=dev, optional=True)
        _expect("w2", w2, (F, D), device=dev)
        _expect("b2", b2, (D,), device=dev, optional=True)
        if not w1.is_cuda:
            raise ValueError("weights must live on a CUDA device")
        self.w1 = pack_cols(w1, t)           # [t][D][Ft]
        self.w2 = pack_rows(w2, t)           # [t][Ft][D]
        self.b1 = None if b1 is None else b1.contiguous()   # [F] == [t][Ft]
        self.b2 = None if b2 is None else b2.contiguous()
        self.device = w1.device
        self.ws = None

    @_nvtx("tp.mlp.forward")
    def forward(self, x, resid=None, out: Optional[Dict] = None):
        d = self.dims
        T, D, F = d.batch * d.seq, d.hidden, d.ffn
        _expect("x", x, (T, D), device=self.device)
        _expect("resid", resid, (T, D), device=self.device, optional=True)
        if out is not None:
            _expect_all(out, {"y": ((T, D), BF16), "a": ((d.t, T, F // d.t), BF16),
                              "h": ((d.t, T, F // d.t), BF16)}, self.device, "out")
        o = out if out is not None else {
            "y": _empty((T, D), device=self.device),
            "a": _empty((d.t, T, F // d.t), device=self.device),
            "h": _empty((d.t, T, F // d.t), device=self.device)}
        mlp_fwd(d, x, self.w1, self.b1, self.w2, self.b2, resid, o["y"], o["a"], o["h"])
        self.saved = (x, o["a"], o["h"])
        return o

    @_nvtx("tp.mlp.backward")
    def backward(self, dy, dres=None, bias_grads=True, out: Optional[Dict] = None):
        d = self.dims
        T, D, F = d.batch * d.seq, d.hidden, d.ffn
        x, a, h = self.saved
        _expect("dy", dy, (T, D), device=self.device)
        _expect("dres", dres, (T, D), device=self.device, optional=True)
        if out is not None:
            _expect_all(out, {"dx": ((T, D), BF16), "dw1": ((d.t, D, F // d.t), BF16),
                              "dw2": ((d.t, F // d.t, D), BF16), "db1": ((F,), BF16),
                              "db2": ((D,), BF16)}, self.device, "out", optional=("db1", "db2"))
        if self.ws is None:
            self.ws = _ws(OP_MLP_BWD, d, self.device)
        g = out if out is not None else {
            "dx": _empty((T, D), device=self.device),
            "dw1": _empty((d.t, D, F // d.t), device=self.device),
            "dw2": _empty((d.t, F // d.t, D), device=self.device),
            "db1": _empty((F,), device=self.device) if bias_grads else None,
            "db2": _empty((D,), device=self.device) if bias_grads else None}
        mlp_bwd(d, x, self.w1, self.w2, a, h, dy, dres, g["dx"], g["dw1"], g["dw2"], g["db1"],
                g["db2"], self.ws)
        return g


class ShardedAttention:
    """Q/K/V split by head, local causal attention, row-parallel Wout + shard sum."""

    def __init__(self, dims: Dims, wqkv, bqkv, wout, bout):
        self.dims = dims
        t, H = dims.t, dims.heads
        D = dims.hidden
        dev = wqkv.device if isinstance(wqkv, torch.Tensor) else None
        _expect("wqkv", wqkv, (D, 3 * D), device=dev)
        _expect("bqkv", bqkv, (3 * D,), device=dev, optional=True)
        _expect("wout", wout, (D, D), device=dev)
        _expect("bout", bout, (D,), device=dev, optional=True)
        if not wqkv.is_cuda:
            raise ValueError("weights must live on a CUDA device")
        self.wqkv = pack_qkv(wqkv, H, t)                                  # [t][D][3Dt]
        self.bqkv = None if bqkv is None else pack_qkv(bqkv, H, t)        # [t][1][3Dt]
        self.wout = pack_rows(wout, t)                                    # [t][Dt][D]
        self.bout = None if bout is None else bout.contiguous()
        self.device = wqkv.device
        self.ws = None
        self.ws_fwd = None

    @_nvtx("tp.attn.forward")
    def forward(self, x, resid=None, out: Optional[Dict] = None):
        d = self.dims
        T, D = d.batch * d.seq, d.hidden
        _expect("x", x, (T, D), device=self.device)
        _expect("resid", resid, (T, D), device=self.device, optional=True)
        if out is not None:
            _expect_all(out, {"y": ((T, D), BF16), "qkv": ((d.t, T, 3 * D // d.t), torch.float16),
                              "o": ((d.t, T, D // d.t), BF16),
                              "lse": ((d.batch, d.heads, d.seq), torch.float32)},
                        self.device, "out")
        o = out if out is not None else {
            "y": _empty((T, D), device=self.device),
            "qkv": _empty((d.t, T, 3 * D // d.t), dtype=torch.float16, device=self.device),
            "o": _empty((d.t, T, D // d.t), device=self.device),
            "lse": _empty((d.batch, d.heads, d.seq), dtype=torch.float32, device=self.device)}
        if self.ws_fwd is None:
            self.ws_fwd = _ws(OP_ATTN_FWD, d, self.device)
        attn_fwd(d, x, self.wqkv, self.bqkv, self.wout, self.bout, resid, o["y"], o["qkv"],
                 o["o"], o["lse"], self.ws_fwd)
        self.saved = (x, o["qkv"], o["o"], o["lse"])
        return o

    @_nvtx("tp.attn.backward")
    def backward(self, dy, dres=None, bias_grads=True, out: Optional[Dict] = None):
        d = self.dims
        T, D = d.batch * d.seq, d.hidden
        x, qkv, o, lse = self.saved
        _expect("dy", dy, (T, D), device=self.device)
        _expect("dres", dres, (T, D), device=self.device, optional=True)
        if out is not None:
            _expect_all(out, {"dx": ((T, D), BF16), "dwqkv": ((d.t, D, 3 * D // d.t), BF16),
                              "dwout": ((d.t, D // d.t, D), BF16),
                              "dbqkv": ((d.t, 1, 3 * D // d.t), BF16), "dbout": ((D,), BF16)},
                        self.device, "out", optional=("dbqkv", "dbout"))
        if self.ws is None:
            self.ws = _ws(OP_ATTN_BWD, d, self.device)
        g = out if out is not None else {
            "dx": _empty((T, D), device=self.device),
            "dwqkv": _empty((d.t, D, 3 * D // d.t), device=self.device),
            "dwout": _empty((d.t, D // d.t, D), device=self.device),
            "dbqkv": _empty((d.t, 1, 3 * D // d.t), device=self.device) if bias_grads else None,
            "dbout": _empty((D,), device=self.device) if bias_grads else None}
        attn_bwd(d, x, self.wqkv, self.wout, qkv, o, lse, dy, dres, g["dx"], g["dwqkv"],
                 g["dbqkv"], g["dwout"], g["dbout"], self.ws)
        return g


LAYER_PARAM_NAMES = ("ln1_g", "ln1_b", "wqkv", "bqkv", "wout", "bout", "ln2_g", "ln2_b",
                     "w1", "b1", "w2", "b2")


class ShardedLayer:
    """Pre-LN layer h = x + Attn(LN1(x)); y = h + MLP(LN2(h)), or with
    placement="post" the post-LN layer h = LN1(x + Attn(x)); y = LN2(h + MLP(h)).

    recompute=True (pre-LN only) keeps nothing but x between forward and
    backward: the forward's intermediates live in its workspace, and the
    backward computes them again before using them."""

    def __init__(self, dims: Dims, p: Dict[str, torch.Tensor], placement: str = "pre",
                 recompute: bool = False):
        if placement not in ("pre", "post"):
            raise ValueError("placement is 'pre' or 'post'")
        if recompute and placement != "pre":
            raise ValueError("recompute is available for the pre-LN layer")
        self.post = placement == "post"
        self.recompute = recompute
        self.dims = dims
        t, H = dims.t, dims.heads
        self.device = p["w1"].device if isinstance(p.get("w1"), torch.Tensor) else None
        _expect_all(p, self._param_spec(), self.device, "p",
                    optional=("bqkv", "bout", "b1", "b2"))
        if not p["w1"].is_cuda:
            raise ValueError("parameters must live on a CUDA device")
        self.p = {
            "ln1_g": p["ln1_g"].contiguous(), "ln1_b": p["ln1_b"].contiguous(),
            "wqkv": pack_qkv(p["wqkv"], H, t),
            "bqkv": None if p.get("bqkv") is None else pack_qkv(p["bqkv"], H, t),
            "wout": pack_rows(p["wout"], t),
            "bout": None if p.get("bout") is None else p["bout"].contiguous(),
            "ln2_g": p["ln2_g"].contiguous(), "ln2_b": p["ln2_b"].contiguous(),
            "w1": pack_cols(p["w1"], t),
            "b1": None if p.get("b1") is None else p["b1"].contiguous(),
            "w2": pack_rows(p["w2"], t),
            "b2": None if p.get("b2") is None else p["b2"].contiguous(),
        }
        self.ws = None
        self.ws_fwd = None

    def _param_spec(self):
        D, F = self.dims.hidden, self.dims.ffn
        return {"ln1_g": ((D,), BF16), "ln1_b": ((D,), BF16), "wqkv": ((D, 3 * D), BF16),
                "bqkv": ((3 * D,), BF16), "wout": ((D, D), BF16), "bout": ((D,), BF16),
                "ln2_g": ((D,), BF16), "ln2_b": ((D,), BF16), "w1": ((D, F), BF16),
                "b1": ((F,), BF16), "w2": ((F, D), BF16), "b2": ((D,), BF16)}

    def _acts_spec(self):
        return {k: (tuple(v.shape), v.dtype) for k, v in self.alloc_acts(meta=True).items()}

    def _grads_spec(self):
        return {k: (tuple(v.shape), v.dtype) for k, v in self.alloc_grads(meta=True).items()}

    def alloc_acts(self, meta=False):
        d = self.dims
        T, D, F, t = d.batch * d.seq, d.hidden, d.ffn, d.t
        f32 = torch.float32
        dev = "meta" if meta else self.device
        f16 = torch.float16
        if self.post:
            return {"z1": _empty((T, D), device=dev), "mean1": _empty((T,), f32, dev),
                    "rstd1": _empty((T,), f32, dev), "qkv": _empty((t, T, 3 * D // t), f16, dev),
                    "o": _empty((t, T, D // t), device=dev),
                    "lse": _empty((d.batch, d.heads, d.seq), f32, dev),
                    "h": _empty((T, D), device=dev), "z2": _empty((T, D), device=dev),
                    "mean2": _empty((T,), f32, dev), "rstd2": _empty((T,), f32, dev),
                    "a": _empty((t, T, F // t), device=dev),
                    "hact": _empty((t, T, F // t), device=dev)}
        return {"u1": _empty((T, D), f16, dev), "mean1": _empty((T,), f32, dev),
                "rstd1": _empty((T,), f32, dev), "qkv": _empty((t, T, 3 * D // t), f16, dev),
                "o": _empty((t, T, D // t), device=dev),
                "lse": _empty((d.batch, d.heads, d.seq), f32, dev),
                "h": _empty((T, D), device=dev), "u2": _empty((T, D), device=dev),
                "mean2": _empty((T,), f32, dev), "rstd2": _empty((T,), f32, dev),
                "a": _empty((t, T, F // t), device=dev), "hact": _empty((t, T, F // t), device=dev),
                # the forward's fp16 copy of Wqkv, reused by the backward
                "wqkv16": _empty((t, D, 3 * D // t), f16, dev)}

    def alloc_grads(self, bias_grads=True, meta=False):
        d = self.dims
        D, F, t = d.hidden, d.ffn, d.t
        dev = "meta" if meta else self.device
        opt = (lambda s: _empty(s, device=dev)) if bias_grads else (lambda s: None)
        return {"dln1_g": opt((D,)), "dln1_b": opt((D,)),
                "dwqkv": _empty((t, D, 3 * D // t), device=dev), "dbqkv": opt((t, 1, 3 * D // t)),
                "dwout": _empty((t, D // t, D), device=dev), "dbout": opt((D,)),
                "dln2_g": opt((D,)), "dln2_b": opt((D,)),
                "dw1": _empty((t, D, F // t), device=dev), "db1": opt((F,)),
                "dw2": _empty((t, F // t, D), device=dev), "db2": opt((D,))}

    def saved_bytes(self) -> int:
        """Bytes of activations held from the forward to the backward (x excluded)."""
        if self.recompute:
            return 0
        return sum(v.numel() * v.element_size() for v in self.alloc_acts(meta=True).values())

    @_nvtx("tp.layer.forward")
    def forward(self, x, acts=None, y=None):
        d = self.dims
        T, D = d.batch * d.seq, d.hidden
        _expect("x", x, (T, D), device=self.device)
        _expect("y", y, (T, D), device=self.device, optional=True)
        if acts is not None:
            _expect_all(acts, self._acts_spec(), self.device, "acts")
        y = y if y is not None else _empty((d.batch * d.seq, d.hidden), device=self.device)
        if self.recompute:
            if self.ws_fwd is None:
                self.ws_fwd = _ws(OP_LAYER_FWD_NOSAVE, d, self.device)
            layer_fwd_nosave(d, x, self.p, y, self.ws_fwd)
            self.saved = (x, None)
            return y, None
        acts = acts if acts is not None else self.alloc_acts()
        if self.ws_fwd is None:
            self.ws_fwd = _ws(OP_POSTLN_FWD if self.post else OP_LAYER_FWD, d, self.device)
        (postln_layer_fwd if self.post else layer_fwd)(d, x, self.p, acts, y, self.ws_fwd)
        self.saved = (x, acts)
        return y, acts

    @_nvtx("tp.layer.backward")
    def backward(self, dy, dx=None, grads=None, bias_grads=True, ready=None):
        """ready (pre-LN, saving layer only): {"mlp", "attn", "ln1"} -> torch.cuda.Event,
        recorded as each group of parameter gradients is enqueued (tp_layer_bwd_notify)."""
        d = self.dims
        x, acts = self.saved
        T, D = d.batch * d.seq, d.hidden
        _expect("dy", dy, (T, D), device=self.device)
        _expect("dx", dx, (T, D), device=self.device, optional=True)
        if grads is not None:
            _expect_all(grads, self._grads_spec(), self.device, "grads",
                        optional=("dln1_g", "dln1_b", "dbqkv", "dbout", "dln2_g", "dln2_b",
                                  "db1", "db2"))
        dx = dx if dx is not None else torch.empty_like(x)
        grads = grads if grads is not None else self.alloc_grads(bias_grads)
        if self.recompute:
            if self.ws is None:
                self.ws = _ws(OP_LAYER_BWD_RECOMPUTE, d, self.device)
            layer_bwd_recompute(d, x, self.p, dy, dx, grads, self.ws)
            return dx, grads
        if self.ws is None:
            self.ws = _ws(OP_POSTLN_BWD if self.post else OP_LAYER_BWD, d, self.device)
        if ready is not None:
            if self.post:
                raise ValueError("gradient-ready events are provided for the pre-LN layer")
            layer_bwd_notify(d, x, self.p, acts, dy, dx, grads, ready, self.ws)
            return dx, grads
        (postln_layer_bwd if self.post else layer_bwd)(d, x, self.p, acts, dy, dx, grads, self.ws)
        return dx, grads
