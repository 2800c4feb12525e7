"""Scalar-loop restatements used to pin the vectorised oracle on tiny shapes.

Every index is walked explicitly, with no matrix product, no reshape and no
transpose, so that a transposed operand, a wrong head/column offset or a
dropped term in the oracle shows up as a mismatch.  Tiny shapes only.
"""
import math


def _gelu(a):
    return 0.5 * a * (1.0 + math.tanh(math.sqrt(2.0 / math.pi) * (a + 0.044715 * a ** 3)))


def mlp_fwd(x, w1, b1, w2, b2):
    T, D = len(x), len(x[0])
    F = len(w1[0])
    y = [[0.0] * D for _ in range(T)]
    for r in range(T):
        h = []
        for j in range(F):
            acc = b1[j]
            for k in range(D):
                acc += x[r][k] * w1[k][j]
            h.append(_gelu(acc))
        for n in range(D):
            acc = b2[n]
            for j in range(F):
                acc += h[j] * w2[j][n]
            y[r][n] = acc
    return y


def layernorm(xrow, gamma, beta, eps):
    D = len(xrow)
    mu = sum(xrow) / D
    var = sum((v - mu) ** 2 for v in xrow) / D
    return [(xrow[i] - mu) / math.sqrt(var + eps) * gamma[i] + beta[i] for i in range(D)]


def attention_fwd(x, wqkv, bqkv, wout, bout, batch, heads, causal=True):
    T, D = len(x), len(x[0])
    S = T // batch
    dh = D // heads

    def proj(r, col):
        acc = bqkv[col]
        for k in range(D):
            acc += x[r][k] * wqkv[k][col]
        return acc

    o = [[0.0] * D for _ in range(T)]
    for b in range(batch):
        for h in range(heads):
            for s in range(S):
                r = b * S + s
                q = [proj(r, h * dh + d) for d in range(dh)]
                keys = range(s + 1) if causal else range(S)
                scores = []
                for sp in keys:
                    rk = b * S + sp
                    kv = [proj(rk, D + h * dh + d) for d in range(dh)]
                    scores.append(sum(q[d] * kv[d] for d in range(dh)) / math.sqrt(dh))
                m = max(scores)
                e = [math.exp(v - m) for v in scores]
                z = sum(e)
                for d in range(dh):
                    acc = 0.0
                    for idx, sp in enumerate(keys):
                        acc += e[idx] / z * proj(b * S + sp, 2 * D + h * dh + d)
                    o[r][h * dh + d] = acc
    y = [[0.0] * D for _ in range(T)]
    for r in range(T):
        for n in range(D):
            acc = bout[n]
            for k in range(D):
                acc += o[r][k] * wout[k][n]
            y[r][n] = acc
    return y
