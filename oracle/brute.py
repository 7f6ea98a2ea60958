"""Loop-only restatement of the decode step for tiny inputs.

TEST INFRASTRUCTURE ONLY.  A second, independent implementation of the same
definitions as ``oracle.mla_oracle`` -- scalar Python loops and ``math``
only, no NumPy matrix routines -- used to pin the vectorised oracle on tiny
shapes (brute force).  It follows "解耦 RoPE（MLA 下）" §五 (append, queries,
scores = content + position, softmax, value aggregation) with the K / V
rebuilt per head as in §七 ``forward_naive``.
"""

from __future__ import annotations

import math


def matvec(W, x):
    """y_r = sum_k W[r][k] x[k] for a row-major ``[out][in]`` weight."""
    return [sum(W[r][k] * x[k] for k in range(len(x))) for r in range(len(W))]


def rope_pairs(v, pos, base, layout):
    """Rotate each frequency pair of ``v`` by pos * base**(-2i/d)."""
    d = len(v)
    out = list(v)
    for i in range(d // 2):
        theta = base ** (-2.0 * i / d)
        a = pos * theta
        if layout == 0:
            j0, j1 = 2 * i, 2 * i + 1
        else:
            j0, j1 = i, i + d // 2
        x0, x1 = v[j0], v[j1]
        out[j0] = x0 * math.cos(a) - x1 * math.sin(a)
        out[j1] = x0 * math.sin(a) + x1 * math.cos(a)
    return out


def rmsnorm(x, gamma, eps):
    ms = sum(t * t for t in x) / len(x)
    inv = 1.0 / math.sqrt(ms + eps)
    return [gamma[i] * x[i] * inv for i in range(len(x))]


def decode_step(h_batch, prior_rows, W, n_heads, d_c, d_rope, d_nope, d_v,
                base=10000.0, eps=1e-6, layout=0, scale=None):
    """Returns (rows_new, q_lat, z, o, u) as nested lists, one entry per sequence."""
    if scale is None:
        scale = 1.0 / math.sqrt(d_nope + d_rope)
    res = []
    for b, h in enumerate(h_batch):
        pos = len(prior_rows[b])
        c = rmsnorm(matvec(W["W_DKV"], h), W["gamma"], eps)
        k_r = rope_pairs(matvec(W["W_KR"], h), pos, base, layout)
        new_row = c + k_r
        rows = [list(r) for r in prior_rows[b]] + [new_row]
        c_q = matvec(W["W_DQ"], h) if W.get("W_DQ") is not None else list(h)
        q_c_all = matvec(W["W_UQ"], c_q)
        q_r_all = matvec(W["W_QR"], c_q)
        q_lat, z, o = [], [], []
        for i in range(n_heads):
            q_c = q_c_all[i * d_nope:(i + 1) * d_nope]
            q_r = rope_pairs(q_r_all[i * d_rope:(i + 1) * d_rope], pos, base, layout)
            w_uk = W["W_UK"][i * d_nope:(i + 1) * d_nope]     # d_nope rows of d_c
            w_uv = W["W_UV"][i * d_v:(i + 1) * d_v]           # d_v rows of d_c
            q_t = [sum(w_uk[a][cc] * q_c[a] for a in range(d_nope)) for cc in range(d_c)]
            q_lat.append(q_t + q_r)
            # un-absorbed scores: K = [W_UK,i c_s ; k_R,s]
            scores = []
            for r in rows:
                k_c = [sum(w_uk[a][cc] * r[cc] for cc in range(d_c)) for a in range(d_nope)]
                s = sum(q_c[a] * k_c[a] for a in range(d_nope))
                s += sum(q_r[j] * r[d_c + j] for j in range(d_rope))
                scores.append(s * scale)
            mx = max(scores)
            e = [math.exp(s - mx) for s in scores]
            tot = sum(e)
            alpha = [t / tot for t in e]
            z.append([sum(alpha[s] * rows[s][cc] for s in range(len(rows))) for cc in range(d_c)])
            vs = [[sum(w_uv[a][cc] * r[cc] for cc in range(d_c)) for a in range(d_v)] for r in rows]
            o.extend(sum(alpha[s] * vs[s][a] for s in range(len(rows))) for a in range(d_v))
        u = matvec(W["W_O"], o) if W.get("W_O") is not None else None
        res.append((new_row, q_lat, z, o, u))
    return res
