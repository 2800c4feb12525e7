"""One shard per GPU: the pre-LN layer as the pages deploy it, driven from the host.

"One Idea, Two Insertions" (explainer) and "How transformer layers actually
decompose" / "Why TP must stay within a node" (blog): GPU i of a t-GPU group
holds shard i of every weight matrix -- columns i*F/t.. of W1, rows of W2,
the heads i*H/t.. of Q/K/V, rows of Wout -- and the shards meet in one
all-reduce per sublayer per direction:

  forward   LN1 -> attention shard -> [sum of O_i Wout_i] -> + bout + x = h
            LN2 -> MLP shard       -> [sum of H_i W2_i]   -> + b2 + h   = y
  backward  MLP shard backward     -> [sum of dA_i W1_i^T]    -> du2; LN2^T -> dh
            attention shard bwd    -> [sum of dqkv_i Wqkv_i^T] -> du1; LN1^T -> dx

The brackets are the four exchanges.  A ``RankLayer`` runs, for its rank,
everything between two exchanges (the phases below) through ``ops``: by
default the rank-local kernels of libtplayer.so (``LibraryRankOps``), which
write each partial in fp32 without bias; the row-parallel bias is added once,
with the residual, when the summed partials are rounded (tp_rowpar_finish).

An exchange turns the list of partial buffers this process owns into the
list of buffers the finish step sums, in rank order:
  * ``AllReduce`` -- one rank per process: an all-reduce (SUM) of the one
    partial over the process group (NCCL over NVLink on GPUs, gloo on CPU);
    the finish then reads that one buffer;
  * ``LocalSum`` -- one process drives all t ranks (several shards on one
    GPU): nothing moves, the finish reads the t partials themselves.

LayerNorm and the replicated tensors (x, h, LN statistics, dy, dh) are
computed identically on every rank, as in the pages' design; the parameter
gradients of the replicated parameters (LayerNorm, bout, b2) come out equal
on every rank, those of the sharded ones are shard-local.
"""
from __future__ import annotations

from typing import Callable, Dict, List, Sequence

import torch

from . import (Dims, RANK_ATTN_BWD, RANK_ATTN_FWD, RANK_MLP_BWD, attn_bwd_rank, attn_fwd_rank,
               layernorm_bwd, layernorm_bwd_workspace_size, layernorm_fwd, layernorm_fwd_f16,
               mlp_bwd_rank, mlp_fwd_rank, rank_workspace_size, rowpar_finish)

BF16, F16, F32 = torch.bfloat16, torch.float16, torch.float32

# Parameter names of one rank: shard-local (sharded matrices and the biases
# split with their columns) and replicated (LayerNorm, row-parallel biases).
SHARDED = ("wqkv", "bqkv", "wout", "w1", "b1", "w2")
REPLICATED = ("ln1_g", "ln1_b", "bout", "ln2_g", "ln2_b", "b2")


def shard_shapes(dims: Dims) -> Dict[str, tuple]:
    """Shapes of rank i's parameters (and of their gradients)."""
    D, F, t = dims.hidden, dims.ffn, dims.t
    Dt, Ft = D // t, F // t
    return {"ln1_g": (D,), "ln1_b": (D,), "wqkv": (D, 3 * Dt), "bqkv": (3 * Dt,),
            "wout": (Dt, D), "bout": (D,), "ln2_g": (D,), "ln2_b": (D,), "w1": (D, Ft),
            "b1": (Ft,), "w2": (Ft, D), "b2": (D,)}


def shard_layer_params(p: Dict[str, torch.Tensor], dims: Dims, rank: int) -> Dict[str, torch.Tensor]:
    """Rank `rank`'s shard of unsharded bf16 CUDA layer parameters, cut with
    the library's layout kernels (each shard copied out on its own)."""
    from .sublayer import pack_cols, pack_qkv, pack_rows
    t, H = dims.t, dims.heads
    out = {k: (None if p.get(k) is None else p[k].contiguous()) for k in REPLICATED}
    out["wqkv"] = pack_qkv(p["wqkv"], H, t)[rank].clone()
    out["bqkv"] = None if p.get("bqkv") is None else pack_qkv(p["bqkv"], H, t)[rank].reshape(-1).clone()
    out["wout"] = pack_rows(p["wout"], t)[rank].clone()
    out["w1"] = pack_cols(p["w1"], t)[rank].clone()
    out["b1"] = None if p.get("b1") is None else p["b1"].reshape(t, -1)[rank].clone()
    out["w2"] = pack_rows(p["w2"], t)[rank].clone()
    return out


# ---------------------------------------------------------------- exchanges
class AllReduce:
    """One rank per process: all-reduce (SUM) of the partial over `group`."""

    def __init__(self, group=None):
        self.group = group
        self.count = 0

    def __call__(self, partials: Sequence[torch.Tensor]) -> List[torch.Tensor]:
        import torch.distributed as dist
        if len(partials) != 1:
            raise ValueError("AllReduce drives exactly one rank per process")
        dist.all_reduce(partials[0], op=dist.ReduceOp.SUM, group=self.group)
        self.count += 1
        return [partials[0]]


class LocalSum:
    """All t ranks in this process: the finish step sums their partials in rank order."""

    def __init__(self):
        self.count = 0

    def __call__(self, partials: Sequence[torch.Tensor]) -> List[torch.Tensor]:
        self.count += 1
        return list(partials)


# ---------------------------------------------------------------- per-rank compute
class LibraryRankOps:
    """The rank-local kernels of libtplayer.so on one GPU; buffers allocated
    once per name and reused across steps."""

    def __init__(self, dims: Dims, device):
        self.dims = dims
        self.device = torch.device(device)
        self._bufs: Dict[str, torch.Tensor] = {}

    def buf(self, key, shape, dtype=BF16):
        b = self._bufs.get(key)
        if b is None or tuple(b.shape) != tuple(shape) or b.dtype != dtype:
            b = torch.empty(shape, dtype=dtype, device=self.device)
            self._bufs[key] = b
        return b

    def _ws(self, key, nbytes):
        return self.buf(key, (max(nbytes, 1),), torch.uint8) if nbytes else None

    def layernorm_fwd(self, key, x, g, b, f16=False):
        d = self.dims
        T, D = x.shape
        y = self.buf(key, (T, D), F16 if f16 else BF16)
        mean, rstd = self.buf(key + ".mean", (T,), F32), self.buf(key + ".rstd", (T,), F32)
        (layernorm_fwd_f16 if f16 else layernorm_fwd)(x, g, b, T, D, d.ln_eps, y, mean, rstd)
        return y, mean, rstd

    def layernorm_bwd(self, key, dy, x, g, mean, rstd, dres, dg, db):
        T, D = x.shape
        dx = self.buf(key, (T, D))
        ws = self._ws(key + ".ws", layernorm_bwd_workspace_size(T, D))
        layernorm_bwd(dy, x, g, mean, rstd, dres, T, D, dx, dg, db, ws)
        return dx

    def attn_fwd(self, x16, wqkv, bqkv, wout):
        d = self.dims
        T, D, t = d.batch * d.seq, d.hidden, d.t
        qkv = self.buf("qkv", (T, 3 * D // t), F16)
        o = self.buf("o", (T, D // t))
        lse = self.buf("lse", (d.batch, d.heads // t, d.seq), F32)
        part = self.buf("part.attn_fwd", (T, D), F32)
        ws = self._ws("ws.attn_fwd", rank_workspace_size(RANK_ATTN_FWD, d))
        attn_fwd_rank(d, None, x16, wqkv, bqkv, wout, qkv, o, lse, part, ws)
        return qkv, o, lse, part

    def attn_bwd(self, x16, wqkv, wout, qkv, o, lse, dy, grads):
        d = self.dims
        T, D = d.batch * d.seq, d.hidden
        part = self.buf("part.attn_bwd", (T, D), F32)
        ws = self._ws("ws.attn_bwd", rank_workspace_size(RANK_ATTN_BWD, d))
        attn_bwd_rank(d, None, x16, wqkv, wout, qkv, o, lse, dy, grads["wqkv"], grads.get("bqkv"),
                      grads["wout"], grads.get("bout"), part, ws)
        return part

    def mlp_fwd(self, x, w1, b1, w2):
        d = self.dims
        T, D, Ft = d.batch * d.seq, d.hidden, d.ffn // d.t
        a, h = self.buf("a", (T, Ft)), self.buf("h", (T, Ft))
        part = self.buf("part.mlp_fwd", (T, D), F32)
        mlp_fwd_rank(d, x, w1, b1, w2, a, h, part)
        return a, h, part

    def mlp_bwd(self, x, w1, w2, a, h, dy, grads):
        d = self.dims
        T, D = d.batch * d.seq, d.hidden
        part = self.buf("part.mlp_bwd", (T, D), F32)
        ws = self._ws("ws.mlp_bwd", rank_workspace_size(RANK_MLP_BWD, d))
        mlp_bwd_rank(d, x, w1, w2, a, h, dy, grads["w1"], grads["w2"], grads.get("b1"),
                     grads.get("b2"), part, ws)
        return part

    def finish(self, key, sources, bias, resid):
        T, D = sources[0].shape
        out = self.buf(key, (T, D))
        rowpar_finish(list(sources), bias, resid, T, D, out)
        return out

    def alloc_grads(self, bias_grads=True):
        shapes = shard_shapes(self.dims)
        optional = ("ln1_g", "ln1_b", "bqkv", "bout", "ln2_g", "ln2_b", "b1", "b2")
        return {k: (None if (k in optional and not bias_grads)
                    else torch.empty(s, dtype=BF16, device=self.device))
                for k, s in shapes.items()}


# ---------------------------------------------------------------- one rank of the layer
class RankLayer:
    """Rank `rank` of t of the pre-LN layer h = x + Attn(LN1(x)), y = h + MLP(LN2(h)).

    `params` holds this rank's shard (``shard_shapes``); `ops` does the
    arithmetic (``LibraryRankOps`` on a GPU).  The phases run the work
    between two exchanges; ``layer_forward`` / ``layer_backward`` sequence
    them for the ranks a process drives."""

    def __init__(self, dims: Dims, rank: int, params: Dict[str, torch.Tensor], ops,
                 grads: Dict[str, torch.Tensor] = None):
        if not 0 <= rank < dims.t:
            raise ValueError(f"rank {rank} outside 0..{dims.t - 1}")
        self.dims, self.rank, self.p, self.ops = dims, rank, params, ops
        self.grads = grads if grads is not None else ops.alloc_grads()
        self.s: Dict[str, torch.Tensor] = {}      # saved activations of this rank

    # forward ----------------------------------------------------------
    def fwd_attention(self, x):
        """LN1 (fp16 output for the fp16 attention products), the shard's
        heads, and the partial O_i Wout_i."""
        p, s = self.p, self.s
        s["x"] = x
        s["u1"], s["mean1"], s["rstd1"] = self.ops.layernorm_fwd("u1", x, p["ln1_g"], p["ln1_b"],
                                                                 f16=True)
        s["qkv"], s["o"], s["lse"], part = self.ops.attn_fwd(s["u1"], p["wqkv"], p.get("bqkv"),
                                                            p["wout"])
        return part

    def fwd_mlp(self, sources):
        """h = sum of the attention partials + bout + x; LN2; the MLP shard and
        its partial H_i W2_i."""
        p, s = self.p, self.s
        s["h"] = self.ops.finish("h", sources, p.get("bout"), s["x"])
        s["u2"], s["mean2"], s["rstd2"] = self.ops.layernorm_fwd("u2", s["h"], p["ln2_g"],
                                                                 p["ln2_b"])
        s["a"], s["hact"], part = self.ops.mlp_fwd(s["u2"], p["w1"], p.get("b1"), p["w2"])
        return part

    def fwd_output(self, sources):
        """y = sum of the MLP partials + b2 + h."""
        return self.ops.finish("y", sources, self.p.get("b2"), self.s["h"])

    # backward ---------------------------------------------------------
    def bwd_mlp(self, dy):
        """The MLP shard's weight gradients (db2 replicated) and the partial dA_i W1_i^T."""
        s = self.s
        s["dy"] = dy
        return self.ops.mlp_bwd(s["u2"], self.p["w1"], self.p["w2"], s["a"], s["hact"], dy,
                                self.grads)

    def bwd_ln2(self, sources):
        """du2 = the summed MLP input gradient; dh = dy + LN2^T(du2) (and LN2's
        parameter gradients, replicated)."""
        p, s, g = self.p, self.s, self.grads
        du2 = self.ops.finish("du2", sources, None, None)
        s["dh"] = self.ops.layernorm_bwd("dh", du2, s["h"], p["ln2_g"], s["mean2"], s["rstd2"],
                                         s["dy"], g.get("ln2_g"), g.get("ln2_b"))

    def bwd_attention(self):
        """The attention shard's gradients (dbout replicated) and the partial dqkv_i Wqkv_i^T."""
        p, s = self.p, self.s
        return self.ops.attn_bwd(s["u1"], p["wqkv"], p["wout"], s["qkv"], s["o"], s["lse"],
                                 s["dh"], self.grads)

    def bwd_input(self, sources):
        """du1 = the summed attention input gradient; dx = dh + LN1^T(du1)."""
        p, s, g = self.p, self.s, self.grads
        du1 = self.ops.finish("du1", sources, None, None)
        return self.ops.layernorm_bwd("dx", du1, s["x"], p["ln1_g"], s["mean1"], s["rstd1"],
                                      s["dh"], g.get("ln1_g"), g.get("ln1_b"))


Exchange = Callable[[Sequence[torch.Tensor]], List[torch.Tensor]]


def layer_forward(ranks: Sequence[RankLayer], x, exchange: Exchange):
    """Forward of the ranks this process drives; returns y per rank (equal on every rank)."""
    sources = exchange([r.fwd_attention(x) for r in ranks])     # attention all-reduce
    sources = exchange([r.fwd_mlp(sources) for r in ranks])     # MLP all-reduce
    return [r.fwd_output(sources) for r in ranks]


def layer_backward(ranks: Sequence[RankLayer], dy, exchange: Exchange, on_grads_ready=None):
    """Backward; returns dx per rank (equal on every rank).  Each rank's
    parameter gradients land in ``rank.grads``.  ``on_grads_ready(group)``,
    if given, is called as soon as the kernels producing a group of gradients
    are enqueued -- the points where a data-parallel reduction of them can
    start: "mlp" after the MLP shard's and LN2's backward (w1, b1, w2, b2, ln2),
    "attn" after the attention shard's (wqkv, bqkv, wout, bout), "ln1" at the
    end: the groups of data_parallel.LAYER_GROUPS, or earlier."""
    sources = exchange([r.bwd_mlp(dy) for r in ranks])          # MLP input-gradient all-reduce
    for r in ranks:
        r.bwd_ln2(sources)
    if on_grads_ready:
        on_grads_ready("mlp")
    sources = exchange([r.bwd_attention() for r in ranks])      # attention all-reduce
    if on_grads_ready:
        on_grads_ready("attn")
    dx = [r.bwd_input(sources) for r in ranks]
    if on_grads_ready:
        on_grads_ready("ln1")
    return dx
