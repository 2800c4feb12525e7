"""Per-rank compute of the one-shard-per-GPU layer on the CPU, in fp64, built
from the oracle's primitives: test infrastructure for the host logic of
tensor_transformer_layer_column_b200.tensor_parallel (phase order, which
tensors the exchanges sum, bias added once, gradient placement) where no GPU
is present.  Same interface as LibraryRankOps; tensors are float64 torch CPU
tensors, so that gloo can all-reduce them.
"""
import numpy as np
import torch

from oracle import core as ocore
from oracle.attention import _heads, _unheads, attn_core_bwd, attn_core_fwd
from oracle import layout as olay
from tensor_transformer_layer_column_b200.tensor_parallel import REPLICATED, shard_shapes

F64 = torch.float64


def _n(t):
    return t.detach().numpy()


def _t(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))


class OracleRankOps:
    def __init__(self, dims):
        self.dims = dims

    def layernorm_fwd(self, key, x, g, b, f16=False):
        y, mean, rstd = ocore.layernorm_fwd(_n(x), _n(g), _n(b), self.dims.ln_eps)
        return _t(y), _t(mean), _t(rstd)

    def layernorm_bwd(self, key, dy, x, g, mean, rstd, dres, dg, db):
        dx, dgam, dbet = ocore.layernorm_bwd(_n(dy), _n(x), _n(g), _n(mean), _n(rstd))
        if dg is not None:
            dg.copy_(_t(dgam))
        if db is not None:
            db.copy_(_t(dbet))
        return _t(dx + (_n(dres) if dres is not None else 0.0))

    def _split(self, qkv):
        d = self.dims
        dt = d.hidden // d.t
        return [_heads(qkv[:, j * dt:(j + 1) * dt], d.batch, d.seq, d.heads // d.t)
                for j in range(3)]

    def attn_fwd(self, x, wqkv, bqkv, wout):
        qkv = _n(x) @ _n(wqkv) + (_n(bqkv) if bqkv is not None else 0.0)
        q, k, v = self._split(qkv)
        o, lse = attn_core_fwd(q, k, v, True)
        o = _unheads(o)
        return _t(qkv), _t(o), _t(lse), _t(o @ _n(wout))

    def attn_bwd(self, x, wqkv, wout, qkv, o, lse, dy, grads):
        d = self.dims
        dyn = _n(dy)
        grads["wout"].copy_(_t(_n(o).T @ dyn))
        do = _heads(dyn @ _n(wout).T, d.batch, d.seq, d.heads // d.t)
        q, k, v = self._split(_n(qkv))
        dqkv = np.concatenate([_unheads(g) for g in attn_core_bwd(q, k, v, do, True)], axis=1)
        grads["wqkv"].copy_(_t(_n(x).T @ dqkv))
        if grads.get("bqkv") is not None:
            grads["bqkv"].copy_(_t(dqkv.sum(axis=0)))
        if grads.get("bout") is not None:
            grads["bout"].copy_(_t(dyn.sum(axis=0)))
        return _t(dqkv @ _n(wqkv).T)

    def mlp_fwd(self, x, w1, b1, w2):
        a = _n(x) @ _n(w1) + (_n(b1) if b1 is not None else 0.0)
        h = ocore.gelu(a)
        return _t(a), _t(h), _t(h @ _n(w2))

    def mlp_bwd(self, x, w1, w2, a, h, dy, grads):
        dyn = _n(dy)
        da = (dyn @ _n(w2).T) * ocore.gelu_grad(_n(a))
        grads["w2"].copy_(_t(_n(h).T @ dyn))
        grads["w1"].copy_(_t(_n(x).T @ da))
        if grads.get("b1") is not None:
            grads["b1"].copy_(_t(da.sum(axis=0)))
        if grads.get("b2") is not None:
            grads["b2"].copy_(_t(dyn.sum(axis=0)))
        return _t(da @ _n(w1).T)

    def finish(self, key, sources, bias, resid):
        out = sources[0].clone()
        for s in sources[1:]:
            out += s
        if bias is not None:
            out += bias
        if resid is not None:
            out += resid
        return out

    def alloc_grads(self):
        return {k: torch.zeros(s, dtype=F64) for k, s in shard_shapes(self.dims).items()}


def rank_params(p64: dict, dims, rank: int) -> dict:
    """Rank `rank`'s shard of unsharded fp64 parameters, cut with the oracle's layout."""
    t = dims.t
    out = {k: _t(p64[k]) for k in REPLICATED}
    out["wqkv"] = _t(olay.shard_qkv(p64["wqkv"], t)[rank])
    out["bqkv"] = _t(olay.shard_qkv(p64["bqkv"][None, :], t)[rank][0])
    out["wout"] = _t(olay.shard_rows(p64["wout"], t)[rank])
    out["w1"] = _t(olay.shard_cols(p64["w1"], t)[rank])
    out["b1"] = _t(p64["b1"].reshape(t, -1)[rank])
    out["w2"] = _t(olay.shard_rows(p64["w2"], t)[rank])
    return out


def expected_rank_grads(g: dict, dims, rank: int) -> dict:
    """The oracle's unsharded gradients cut to rank `rank`'s shard."""
    t = dims.t
    return {
        "ln1_g": g["dln1_g"], "ln1_b": g["dln1_b"], "bout": g["dbout"],
        "ln2_g": g["dln2_g"], "ln2_b": g["dln2_b"], "b2": g["db2"],
        "wqkv": olay.shard_qkv(g["dwqkv"], t)[rank],
        "bqkv": olay.shard_qkv(g["dbqkv"][None, :], t)[rank][0],
        "wout": olay.shard_rows(g["dwout"], t)[rank],
        "w1": olay.shard_cols(g["dw1"], t)[rank],
        "b1": g["db1"].reshape(t, -1)[rank],
        "w2": olay.shard_rows(g["dw2"], t)[rank],
    }
