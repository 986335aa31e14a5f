"""Pure-Python brute-force forms of the scoring steps, for tiny inputs only.

Independent of ``oracle/`` (no shared code): plain lists, explicit loops and
``math.exp``.  Used to pin the oracle, never the CUDA path directly.
"""
import math


def pool_padded(rows, mask, chunk):
    """Masked mean over groups of ``chunk`` rows of a padded document.

    ``rows``: list of H-lists (padded length), ``mask``: list of 0/1 of the same
    length.  A group whose mask is all zero yields no vector."""
    out = []
    H = len(rows[0]) if rows else 0
    for g0 in range(0, len(rows), chunk):
        cnt = 0
        acc = [0.0] * H
        for t in range(g0, min(g0 + chunk, len(rows))):
            if mask[t]:
                cnt += 1
                for j in range(H):
                    acc[j] += rows[t][j]
        if cnt:
            out.append([a / cnt for a in acc])
    return out


def matvec_rows(x, w):
    """y[i][o] = sum_k x[i][k] * w[o][k]  (w stored [out][in])."""
    return [[sum(xi[k] * wo[k] for k in range(len(xi))) for wo in w] for xi in x]


def attention_concat(q, ks, vs, kc, vc, scale):
    """Merged attention by explicit concatenation, one row at a time.

    q: [Lq][n_q][D]; ks, vs: [Lq][n_kv][D]; kc, vc: [Nc][n_kv][D].
    Row i of head h attends to [ks[0..i] ; kc[0..Nc-1]] of KV head h // G.
    Returns (o [Lq][n_q][D], lse [Lq][n_q])."""
    Lq = len(q)
    n_q = len(q[0])
    D = len(q[0][0])
    n_kv = len(ks[0]) if ks else len(kc[0])
    G = n_q // n_kv
    o = [[[0.0] * D for _ in range(n_q)] for _ in range(Lq)]
    lse = [[0.0] * n_q for _ in range(Lq)]
    for i in range(Lq):
        for h in range(n_q):
            g = h // G
            keys = [ks[j][g] for j in range(i + 1)] + [kc[c][g] for c in range(len(kc))]
            vals = [vs[j][g] for j in range(i + 1)] + [vc[c][g] for c in range(len(vc))]
            logits = [scale * sum(q[i][h][t] * k[t] for t in range(D)) for k in keys]
            m = max(logits)
            e = [math.exp(s - m) for s in logits]
            z = sum(e)
            for t in range(D):
                o[i][h][t] = sum(e[j] * vals[j][t] for j in range(len(vals))) / z
            lse[i][h] = m + math.log(z)
    return o, lse


def softmax2_first(y, n):
    """softmax([y, n])[0] computed as a plain two-entry softmax."""
    m = max(y, n)
    a = math.exp(y - m)
    b = math.exp(n - m)
    return a / (a + b)
