"""Pure-Python, loop-only restatement of the path for tiny shapes.

Used only as a pin for the numpy oracle (brute force on tiny inputs): every
product is an explicit loop over scalars with ``math.fsum`` accumulation, no
numpy, no matrix primitives, so a transposed operand, a broadcast over the
wrong axis or a dropped term in the oracle shows up as a mismatch.
"""
from __future__ import annotations

import math


def linear(xrows, w, b=None):
    """xrows: list of rows (len in); w: list of out-rows (len in); b: list or None."""
    out = []
    for x in xrows:
        row = []
        for o, wr in enumerate(w):
            acc = math.fsum(xi * wi for xi, wi in zip(x, wr))
            row.append(acc + (b[o] if b is not None else 0.0))
        out.append(row)
    return out


def rmsnorm(xrows, g, eps):
    out = []
    for x in xrows:
        ms = math.fsum(v * v for v in x) / len(x)
        r = 1.0 / math.sqrt(ms + eps)
        out.append([v * r * gi for v, gi in zip(x, g)])
    return out


def rope_vec(v, p, base):
    hd = len(v)
    half = hd // 2
    out = list(v)
    for i in range(half):
        ang = p * base ** (-2.0 * i / hd)
        c, s = math.cos(ang), math.sin(ang)
        out[i] = v[i] * c - v[i + half] * s
        out[i + half] = v[i + half] * c + v[i] * s
    return out


def heads(rows, n, hd):
    """rows [T][n*hd] -> [n][T][hd]"""
    return [[r[h * hd:(h + 1) * hd] for r in rows] for h in range(n)]


def attend(q, k, v, allowed):
    """q [nq][Tq][hd], k/v [nkv][Tk][hd], allowed(i, j) -> bool; returns rows [Tq][nq*hd]."""
    nq, nkv = len(q), len(k)
    hd = len(q[0][0])
    Tq = len(q[0])
    out = [[0.0] * (nq * hd) for _ in range(Tq)]
    for h in range(nq):
        g = h * nkv // nq
        for i in range(Tq):
            scores = []
            for j in range(len(k[g])):
                if allowed(i, j):
                    scores.append((j, math.fsum(a * b for a, b in zip(q[h][i], k[g][j])) / math.sqrt(hd)))
            m = max(sc for _, sc in scores)
            ws = [(j, math.exp(sc - m)) for j, sc in scores]
            z = math.fsum(w for _, w in ws)
            for d in range(hd):
                out[i][h * hd + d] = math.fsum(w * v[g][j][d] for j, w in ws) / z
    return out


def add(a, b):
    return [[x + y for x, y in zip(ra, rb)] for ra, rb in zip(a, b)]


def swiglu(y, wg, wu, wd):
    g = linear(y, wg)
    u = linear(y, wu)
    h = [[gv / (1.0 + math.exp(-gv)) * uv for gv, uv in zip(gr, ur)] for gr, ur in zip(g, u)]
    return linear(h, wd)


def tolist(W):
    return {k: v.tolist() for k, v in W.items()}


def prefill(W, s, embeds, valid):
    """Returns K, V as [layers][L][kv_heads*hd] lists."""
    L = len(embeds)
    hd = s.head_dim
    pos, c = [], 0
    for j in range(L):
        c += 1 if valid[j] else 0
        pos.append(c - 1)
    x = [list(r) for r in embeds]
    Ks, Vs = [], []
    for l in range(s.p_layers):
        p = f"p{l}."
        y = rmsnorm(x, W[p + "in_norm"], s.rms_eps)
        q = heads(linear(y, W[p + "wq"]), s.p_heads, hd)
        k = heads(linear(y, W[p + "wk"]), s.p_kv_heads, hd)
        v = heads(linear(y, W[p + "wv"]), s.p_kv_heads, hd)
        q = [[rope_vec(q[h][i], pos[i], s.rope_base) for i in range(L)] for h in range(s.p_heads)]
        k = [[rope_vec(k[h][i], pos[i], s.rope_base) for i in range(L)] for h in range(s.p_kv_heads)]
        Ks.append([[k[h][i][d] for h in range(s.p_kv_heads) for d in range(hd)] for i in range(L)])
        Vs.append([[v[h][i][d] for h in range(s.p_kv_heads) for d in range(hd)] for i in range(L)])
        o = attend(q, k, v, lambda i, j: bool(valid[j]))
        x = add(x, linear(o, W[p + "wo"]))
        x = add(x, swiglu(rmsnorm(x, W[p + "post_norm"], s.rms_eps), W[p + "wg"], W[p + "wu"], W[p + "wd"]))
    return Ks, Vs


def velocity(W, s, x, t, Ks, Vs, valid):
    H = len(x)
    De = s.e_width
    hd = s.head_dim
    a = linear(x, W["w_in"], W["b_in"])
    half = De // 2
    e = [0.0] * De
    for i in range(half):
        period = s.t_min_period * (s.t_max_period / s.t_min_period) ** (i / (half - 1))
        e[i] = math.sin(2.0 * math.pi * t / period)
        e[half + i] = math.cos(2.0 * math.pi * t / period)
    h = linear([ar + e for ar in a], W["w_t1"], W["b_t1"])
    h = [[v / (1.0 + math.exp(-v)) for v in r] for r in h]
    r = linear(h, W["w_t2"], W["b_t2"])
    for l in range(s.e_layers):
        p = f"e{l}."
        y = rmsnorm(r, W[p + "in_norm"], s.rms_eps)
        q = heads(linear(y, W[p + "wq"]), s.e_heads, hd)
        if l % 2 == 0:
            k = heads(linear(y, W[p + "wk"]), s.e_kv_heads, hd)
            v = heads(linear(y, W[p + "wv"]), s.e_kv_heads, hd)
            q = [[rope_vec(q[hh][i], i, s.rope_base) for i in range(H)] for hh in range(s.e_heads)]
            k = [[rope_vec(k[hh][i], i, s.rope_base) for i in range(H)] for hh in range(s.e_kv_heads)]
            o = attend(q, k, v, lambda i, j: j <= i)
        else:
            k = heads(linear(Ks[l], W[p + "wk"]), s.e_kv_heads, hd)
            v = heads(linear(Vs[l], W[p + "wv"]), s.e_kv_heads, hd)
            o = attend(q, k, v, lambda i, j: bool(valid[j]))
        r = add(r, linear(o, W[p + "wo"]))
        r = add(r, swiglu(rmsnorm(r, W[p + "post_norm"], s.rms_eps), W[p + "wg"], W[p + "wu"], W[p + "wd"]))
    return linear(rmsnorm(r, W["final_norm"], s.rms_eps), W["w_out"], W["b_out"])


def sample(W, s, embeds, valid, noise, n_steps):
    Ks, Vs = prefill(W, s, embeds, valid)
    x = [list(r) for r in noise]
    dt = -1.0 / n_steps
    for k in range(n_steps):
        v = velocity(W, s, x, 1.0 + k * dt, Ks, Vs, valid)
        x = [[xi + dt * vi for xi, vi in zip(xr, vr)] for xr, vr in zip(x, v)]
    return Ks, Vs, x
