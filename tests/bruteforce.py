"""Pure-Python brute force of the path's definitions, for tiny inputs only.

Written independently of `oracle/` (lists, loops and the `math` module; no numpy)
so that the oracle can be checked against a second implementation. Sources are
the same pages: the Qwen2.5-1M explainer (DCA patterns, vertical-slash steps,
chunked prefill, attention recall) and the rotary code of the long-context
essay (section 2.4).
"""
from __future__ import annotations

import math


def bf16(x: float) -> float:
    """Nearest bfloat16 (8 significant bits), ties to even, via frexp."""
    if x == 0.0:
        return 0.0
    m, ex = math.frexp(x)  # x = m * 2**ex, 0.5 <= |m| < 1
    q = round(m * 256.0)  # Python rounds half to even
    return math.ldexp(q / 256.0, ex)


def rope_row(x, p, base, rnd=True):
    d = len(x)
    h = d // 2
    y = [0.0] * d
    for m in range(h):
        th = 1.0 / math.pow(base, 2.0 * m / d)
        c, s = math.cos(p * th), math.sin(p * th)
        y[m] = x[m] * c - x[m + h] * s
        y[m + h] = x[m + h] * c + x[m] * s
    return [bf16(t) for t in y] if rnd else y


def dot(a, b):
    return sum(x * y for x, y in zip(a, b))


def estimate(q_rows, k, e, base, scale):
    nr = len(q_rows)
    rows = list(range(e - nr, e))
    kr = [rope_row(k[j], j, base) for j in range(e)]
    lse, A = [], []
    for r, i in enumerate(rows):
        qi = rope_row(q_rows[r], i, base)
        s = [scale * dot(qi, kr[j]) for j in range(i + 1)]
        mx = max(s)
        z = sum(math.exp(t - mx) for t in s)
        l = mx + math.log(z)
        lse.append(l)
        A.append([math.exp(t - l) for t in s] + [0.0] * (e - i - 1))
    vert = [sum(A[r][j] for r in range(nr)) for j in range(e)]
    slash = [0.0] * e
    for r, i in enumerate(rows):
        for j in range(i + 1):
            slash[i - j] += A[r][j]
    return lse, vert, slash, A


def topk(score, k):
    order = sorted(range(len(score)), key=lambda j: (-score[j], j))
    return sorted(order[: min(k, len(score))])


def select(vert, slash, kv, ks):
    sl = list(slash)
    sl[0] = math.inf
    return topk(vert, kv), topk(sl, ks)


def covered(i, j, Vset, Sset):
    return j <= i and (j in Vset or (i - j) in Sset)


def recall(A, rows, V, S):
    Vs, Ss = set(V), set(S)
    tot = 0.0
    for r, i in enumerate(rows):
        tot += sum(A[r][j] for j in range(i + 1) if covered(i, j, Vs, Ss))
    return tot / len(rows)


def refine(A, rows, vert, slash, kv, ks, tau, max_iters=64):
    e = len(vert)
    kv, ks = min(kv, e), min(ks, e)
    it = 0
    while True:
        V, S = select(vert, slash, kv, ks)
        rc = recall(A, rows, V, S)
        if rc >= tau or (kv >= e and ks >= e) or it == max_iters:
            return kv, ks, V, S, rc
        kv, ks = min(2 * kv, e), min(2 * ks, e)
        it += 1


def dca_pos(i, j, C, W):
    """Positions under the three DCA patterns with chunk stride S = C - W."""
    S = C - W
    pk = j % S
    if i // S == j // S:
        pq = i % S
    elif i // S == j // S + 1:
        pq = min(i % S + S, C - 1)
    else:
        pq = C - 1
    return pq, pk


def attention(q_rows, rows, k, v, e, V, S, base, scale, dca=None):
    Vs, Ss = set(V), set(S)
    out, lses = [], []
    for r, i in enumerate(rows):
        js = [j for j in range(i + 1) if covered(i, j, Vs, Ss)]
        s = []
        for j in js:
            if dca is None:
                pq, pk = i, j
            else:
                pq, pk = dca_pos(i, j, *dca)
            s.append(scale * dot(rope_row(q_rows[r], pq, base), rope_row(k[j], pk, base)))
        mx = max(s)
        w = [math.exp(t - mx) for t in s]
        z = sum(w)
        lses.append(mx + math.log(z))
        d = len(v[0])
        out.append([bf16(sum(w[n] * v[js[n]][c] for n in range(len(js))) / z) for c in range(d)])
    return out, lses
