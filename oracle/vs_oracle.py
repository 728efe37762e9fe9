"""Float64 CPU oracle of the Qwen2.5-1M sparse prefill path (TEST INFRASTRUCTURE ONLY).

Sources (pages, with the section each function follows):
  [QW]  "Paper explainer: Qwen2.5-1M" (0h-n0.github.io/posts/paper-2501-15383),
        sections "Length Extrapolation" (DCA's three patterns), "Sparse Attention"
        (vertical-slash steps), "Chunked Prefill" (32K chunks, last 64 queries of
        each chunk), "Sparsity Refinement" (attention recall formulas) and
        "Algorithm: integrating DCA and sparse attention" (the chunk loop; select
        with continuous positions, attend with DCA positions).
  [LC]  "Long-context architecture" essay (deepseekmodel.com), section 2.4
        (the rotary code: inverse frequencies 1/base^(2i/dim), cos/sin of
        position x frequency duplicated over both halves, rotate_half).

Conventions: tensors are numpy float64 arrays holding bf16 values; heads are
handled by the caller one at a time (GQA: query head h reads KV head h // g).
Nothing here is blocked, fused or reordered beyond what the definitions state,
except `attention_rows`, which evaluates rows in blocks of rows (the same
arithmetic per row as `attention_rows_dense`; the equality is a pinned test).

Parity pins (tests/test_oracle_pins.py, all `not gpu`): pure-Python brute force
for every function on tiny inputs; row softmax sums to 1; vertical and slash
mass both equal the number of estimation rows; the full mask equals textbook
dense causal attention; DCA with C >= N equals plain RoPE; DCA's three
statements on random pairs; RoPE relativity; the recall identity and its
monotonicity; top-k against a stable lexicographic sort; chunked == unchunked
under the full mask; MHA and explicit KV repetition for GQA.
Parity unpinned by the pages (readings fixed here, none of them stated there): the DCA local
window W = C/32, doubling both budgets per refinement step, the mean over the
estimation rows as the head's recall, the forced slash offset 0.
"""
from __future__ import annotations

import math
from typing import Optional

import numpy as np

_NEG_INF = -np.inf


# ----------------------------------------------------------------------------- numerics
def bf16_rne(x) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (ties to even), returned as
    float64. bfloat16 keeps 8 significant bits and float32's exponent range;
    rounding drops the low 45 of float64's 52 fraction bits."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    ax = np.abs(x)
    if np.any((ax > 0) & (ax < 2.0 ** -126)):
        raise ValueError("value in the bfloat16 subnormal range")
    b = x.view(np.uint64)
    lsb = (b >> np.uint64(45)) & np.uint64(1)
    r = (b + np.uint64((1 << 44) - 1) + lsb) & np.uint64(~((1 << 45) - 1) & 0xFFFFFFFFFFFFFFFF)
    return r.view(np.float64)


# ----------------------------------------------------------------------------- RoPE  [LC 2.4]
def inv_freq(d: int, base: float) -> np.ndarray:
    """theta_m = 1 / base^(2m/d), m = 0 .. d/2-1, in float64 ([LC] 2.4)."""
    return np.array([1.0 / math.pow(base, (2.0 * m) / d) for m in range(d // 2)], dtype=np.float64)


def rope(x: np.ndarray, pos, base: float, round_bf16: bool = True) -> np.ndarray:
    """Rotate rows of x (n x d) to positions pos (n,), rotate-half convention:
    y[m] = x[m] cos(p theta_m) - x[m + d/2] sin(p theta_m),
    y[m + d/2] = x[m + d/2] cos(p theta_m) + x[m] sin(p theta_m)   ([LC] 2.4).
    Angles and products in float64; the result is rounded once to bf16, the
    operand precision the tensor cores consume."""
    x = np.asarray(x, dtype=np.float64)
    n, d = x.shape
    half = d // 2
    p = np.asarray(pos, dtype=np.float64).reshape(n, 1)
    ang = p * inv_freq(d, base).reshape(1, half)
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[:, :half], x[:, half:]
    y = np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=1)
    return bf16_rne(y) if round_bf16 else y


# ----------------------------------------------------------------------------- DCA  [QW Length Extrapolation]
def dca_q_position(i: int, cls: int, C: int, W: int) -> int:
    """Query position for a key in class cls (0 intra, 1 successive, 2 inter).
    Chunks of stride S = C - W; r(i) = i mod S.
      intra:      the original in-chunk position r(i)
      successive: r(i) + S (exact relative distance inside the local window),
                  clipped to C - 1 beyond it
      inter:      C - 1 (the largest distance the pretraining length allows)."""
    S = C - W
    r = i % S
    if cls == 0:
        return r
    if cls == 1:
        return min(r + S, C - 1)
    return C - 1


def dca_positions(i: int, j, C: int, W: int):
    """(query position, key position) arrays for query i and keys j <= i under DCA
    ([QW] Length Extrapolation, three attention patterns). Key position r(j)."""
    j = np.asarray(j, dtype=np.int64)
    S = C - W
    bi, bj = i // S, j // S
    cls = np.where(bj == bi, 0, np.where(bj == bi - 1, 1, 2))
    pq = np.array([dca_q_position(i, int(c), C, W) for c in (0, 1, 2)], dtype=np.int64)[cls]
    return pq, j % S


# ----------------------------------------------------------------------------- estimation  [QW Sparse Attention, Chunked Prefill]
def estimate(q_rows: np.ndarray, k: np.ndarray, e: int, base: float, scale: float,
             k_rot: Optional[np.ndarray] = None):
    """Attention of the chunk's last queries against every visible key, with
    continuous positions ([QW] "Algorithm": select with continuous positions;
    "Chunked Prefill": the last 64 queries of each chunk).

    q_rows: (nr x d) pre-RoPE queries at positions e-nr .. e-1; k: (>= e x d)
    pre-RoPE keys of the matching KV head. Causal: query i sees keys j <= i.
    k_rot: optionally rope(k, arange, base) already computed (rows >= e), so that
    a caller estimating many chunks of one KV head rotates its keys once; the
    same rows, the same arithmetic.
    Returns lse (nr,), vert (e,) with vert[j] = sum_i A_ij, and slash (e,) with
    slash[dd] = sum_i A_{i, i-dd}, where A = row softmax of the scaled scores."""
    nr = q_rows.shape[0]
    rows = np.arange(e - nr, e)
    qr = rope(q_rows, rows, base)
    kr = rope(k[:e], np.arange(e), base) if k_rot is None else k_rot[:e]
    s = scale * (qr @ kr.T)
    cols = np.arange(e)
    s = np.where(cols[None, :] <= rows[:, None], s, _NEG_INF)
    mx = s.max(axis=1, keepdims=True)
    lse = (mx + np.log(np.exp(s - mx).sum(axis=1, keepdims=True)))[:, 0]
    a = np.exp(s - lse[:, None])
    vert = a.sum(axis=0)
    slash = np.zeros(e, dtype=np.float64)
    for r in range(nr):
        i = rows[r]
        slash[: i + 1] += a[r, i::-1]  # offset dd = i - j for j = i, i-1, ..., 0
    return lse, vert, slash, a


def estimate_probs_dca(q_rows: np.ndarray, k: np.ndarray, e: int, base: float, scale: float,
                       dca: tuple):
    """The estimation rows' attention at DCA positions (dca = (C, W)): the softmax
    the prefill applies to these rows over all keys j <= i ([QW] Length
    Extrapolation: each (query, key) pair scored at the positions of its class).
    Used by the recall-at-DCA-positions variant of refinement; selection itself
    keeps the continuous positions of `estimate`. Returns (lse (nr,), A (nr, e))."""
    C, W = dca
    nr = q_rows.shape[0]
    rows = np.arange(e - nr, e)
    kr = rope(k[:e], np.arange(e) % (C - W), base)
    s = np.full((nr, e), _NEG_INF)
    for r, i in enumerate(rows):
        j = np.arange(i + 1)
        pq, _ = dca_positions(int(i), j, C, W)
        qv = {int(p): rope(q_rows[r : r + 1], np.array([p]), base)[0] for p in np.unique(pq)}
        qj = np.stack([qv[int(p)] for p in pq])
        s[r, : i + 1] = scale * np.einsum("jd,jd->j", qj, kr[: i + 1])
    mx = s.max(axis=1, keepdims=True)
    lse = (mx + np.log(np.exp(s - mx).sum(axis=1, keepdims=True)))[:, 0]
    return lse, np.exp(s - lse[:, None])


# ----------------------------------------------------------------------------- selection  [QW Sparse Attention]
def ranking(score: np.ndarray) -> np.ndarray:
    """All indices ranked by (score descending, index ascending)."""
    n = score.shape[0]
    return np.lexsort((np.arange(n), -score))


def topk_sorted(score: np.ndarray, k: int, order: Optional[np.ndarray] = None) -> np.ndarray:
    """Indices of the k largest scores, ranked by (score descending, index
    ascending), returned in ascending index order. order: ranking(score) when
    the caller has it already (the same ranking, computed once)."""
    n = score.shape[0]
    k = min(int(k), n)
    if order is None:
        order = ranking(score)
    return np.sort(order[:k]).astype(np.int64)


def kth_score(score: np.ndarray, k: int, order: Optional[np.ndarray] = None) -> float:
    """The score of the k-th ranked element (k capped at the length): the
    boundary of the top-k set."""
    n = score.shape[0]
    k = min(int(k), n)
    if order is None:
        order = ranking(score)
    return float(score[order[k - 1]])


def slash_scores(slash: np.ndarray) -> np.ndarray:
    """The slash scores as ranked by the selection: offset 0 (the main
    diagonal) forced in front of every other offset."""
    sl = slash.copy()
    sl[0] = np.inf
    return sl


def select_orders(vert: np.ndarray, slash: np.ndarray):
    """(ranking of vert, ranking of the slash scores with offset 0 forced)."""
    return ranking(vert), ranking(slash_scores(slash))


def select(vert: np.ndarray, slash: np.ndarray, kv: int, ks: int, orders=None):
    """Critical tokens of the vertical-slash pattern ([QW] Sparse Attention, step
    3): the kv columns with the largest vertical scores and the ks diagonal
    offsets with the largest slash scores. Offset 0 (the main diagonal) is
    always selected. Both lists ascending. orders: select_orders(vert, slash)
    when the caller has them already."""
    ov, osl = orders if orders is not None else (None, None)
    return topk_sorted(vert, kv, ov), topk_sorted(slash_scores(slash), ks, osl)


def membership(e: int, idx: np.ndarray) -> np.ndarray:
    m = np.zeros(e, dtype=bool)
    m[idx] = True
    return m


def recall(a: np.ndarray, rows: np.ndarray, inV: np.ndarray, inS: np.ndarray) -> float:
    """Attention recall of the estimation rows ([QW] Sparsity Refinement):
    per row, exp(lse_sparse - lse_full) = sum of A_ij over the selected keys;
    the head's recall is the mean over the rows."""
    tot = 0.0
    for r, i in enumerate(rows):
        i = int(i)
        # keys j = 0 .. i: column j selected, or offset i - j selected (inS read backwards
        # from offset i down to offset 0)
        sel = inV[: i + 1] | inS[i::-1]
        tot += a[r, : i + 1][sel].sum()
    return tot / len(rows)


def refine(a: np.ndarray, rows: np.ndarray, vert: np.ndarray, slash: np.ndarray, kv: int, ks: int,
           tau: float, max_iters: int = 64):
    """Sparsity refinement ([QW] Sparsity Refinement): while the head's recall is
    below tau and a budget can still grow, double both budgets (capped at the
    number of visible keys) and select again. Returns the final (kv, ks), the
    sets, the recall and the per-step recall trace."""
    e = vert.shape[0]
    kv, ks = min(int(kv), e), min(int(ks), e)
    trace = []
    orders = select_orders(vert, slash)  # the ranking does not change between steps
    for it in range(max_iters + 1):
        V, S = select(vert, slash, kv, ks, orders)
        rc = recall(a, rows, membership(e, V), membership(e, S))
        trace.append((kv, ks, rc))
        if rc >= tau or (kv >= e and ks >= e) or it == max_iters:
            break
        kv, ks = min(2 * kv, e), min(2 * ks, e)
    return kv, ks, V, S, rc, trace


# ----------------------------------------------------------------------------- attention  [QW Sparse Attention step 4; Algorithm]
def _key_positions(e: int, dca: Optional[tuple]) -> np.ndarray:
    if dca is None:
        return np.arange(e)
    C, W = dca
    return np.arange(e) % (C - W)


def attention_rows_dense(q_rows: np.ndarray, rows: np.ndarray, k: np.ndarray, v: np.ndarray, e: int,
                         inV: np.ndarray, inS: np.ndarray, base: float, scale: float,
                         dca: Optional[tuple] = None):
    """Literal definition, one query row at a time: O_i = sum over the selected
    keys j <= i (j a vertical column or i - j a slash offset) of softmax(s_ij) v_j,
    with s_ij from RoPE'd q_i and k_j at DCA positions (dca = (C, W)) or at
    continuous positions. Returns (bf16-rounded outputs, lse) in float64."""
    kr = rope(k[:e], _key_positions(e, dca), base)
    out = np.zeros((len(rows), v.shape[1]))
    lse = np.zeros(len(rows))
    for r, i in enumerate(rows):
        j = np.arange(i + 1)
        sel = inV[: i + 1] | inS[i - j]
        js = j[sel]
        if dca is None:
            pq = np.full(js.shape, i)
        else:
            pq, _ = dca_positions(int(i), js, *dca)
        s = np.empty(js.shape[0])
        for p in np.unique(pq):
            qi = rope(q_rows[r : r + 1], [p], base)[0]
            m = pq == p
            s[m] = scale * (kr[js[m]] @ qi)
        mx = s.max()
        w = np.exp(s - mx)
        lse[r] = mx + np.log(w.sum())
        out[r] = (w / w.sum()) @ v[js]
    return bf16_rne(out), lse


def attention_rows(q_rows: np.ndarray, rows: np.ndarray, k: np.ndarray, v: np.ndarray, e: int,
                   inV: np.ndarray, inS: np.ndarray, base: float, scale: float,
                   dca: Optional[tuple] = None, block: int = 128, k_rot: Optional[np.ndarray] = None,
                   round_out: bool = True):
    """Same arithmetic as `attention_rows_dense`, evaluated for blocks of rows at
    a time over the keys the block can see (masked entries are -inf and
    contribute exactly zero). k_rot: optionally the keys already rotated to their
    key positions (rope(k, _key_positions(n, dca), base), rows >= e). round_out:
    False returns the float64 outputs before their final rounding to bf16."""
    rows = np.asarray(rows, dtype=np.int64)
    kr = rope(k[:e], _key_positions(e, dca), base) if k_rot is None else k_rot[:e]
    out = np.zeros((len(rows), v.shape[1]))
    lse = np.zeros(len(rows))
    for b0 in range(0, len(rows), block):
        rb = rows[b0 : b0 + block]
        qb = q_rows[b0 : b0 + block]
        hi = int(rb.max()) + 1
        j = np.arange(hi)
        diff = rb[:, None] - j[None, :]
        sel = (diff >= 0) & (inV[None, :hi] | inS[np.clip(diff, 0, e - 1)])
        if dca is None:
            s = scale * (rope(qb, rb, base) @ kr[:hi].T)
        else:
            C, W = dca
            S = C - W
            cls = np.where(j[None, :] // S == rb[:, None] // S, 0,
                           np.where(j[None, :] // S == rb[:, None] // S - 1, 1, 2))
            s = np.empty(diff.shape)
            for c in (0, 1, 2):
                pq = np.array([dca_q_position(int(i), c, C, W) for i in rb])
                sc = scale * (rope(qb, pq, base) @ kr[:hi].T)
                s = np.where(cls == c, sc, s)
        s = np.where(sel, s, _NEG_INF)
        mx = s.max(axis=1, keepdims=True)
        w = np.exp(s - mx)
        den = w.sum(axis=1, keepdims=True)
        lse[b0 : b0 + block] = (mx + np.log(den))[:, 0]
        out[b0 : b0 + block] = (w / den) @ v[:hi]
    return (bf16_rne(out) if round_out else out), lse


def key_positions(e: int, dca: Optional[tuple] = None) -> np.ndarray:
    """Positions the keys 0 .. e-1 are rotated to in attention: j, or j mod (C - W)
    under DCA ([QW] Length Extrapolation)."""
    return _key_positions(e, dca)


# ----------------------------------------------------------------------------- the chunk loop  [QW Algorithm; Chunked Prefill]
def calibrate(q: np.ndarray, k: np.ndarray, *, chunk: int, last_q: int, kv_budget: int, ks_budget: int,
              tau: float, base: float, scale: Optional[float] = None, max_iters: int = 64, heads=None):
    """Offline form of sparsity refinement ([QW] Chunked Prefill, the sparsity-
    refinement passage: the budgets are improved once on a calibration sequence).
    Reading: every chunk of the calibration sequence is refined from the base
    budgets per head, and a head keeps the largest refined budgets over the chunks
    (those that reach tau on every chunk). Returns (kv, ks), one int per head."""
    hq, n, d = q.shape
    g = hq // k.shape[0]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    heads = list(range(hq)) if heads is None else list(heads)
    kv_c = {h: 0 for h in heads}
    ks_c = {h: 0 for h in heads}
    for cs in range(0, n, chunk):
        e = min(cs + chunk, n)
        nr = min(last_q, e - cs)
        est_rows = np.arange(e - nr, e)
        for h in heads:
            _, vert, slash, a = estimate(q[h, e - nr : e], k[h // g], e, base, scale)
            kv, ks, _, _, _, _ = refine(a, est_rows, vert, slash, kv_budget, ks_budget, tau, max_iters)
            kv_c[h], ks_c[h] = max(kv_c[h], kv), max(ks_c[h], ks)
    return [kv_c[h] for h in heads], [ks_c[h] for h in heads]


def layer_prefill(q: np.ndarray, k: np.ndarray, v: np.ndarray, *, chunk: int, last_q: int,
                  kv_budget, ks_budget, tau: Optional[float], base: float,
                  scale: Optional[float] = None, dca: Optional[tuple] = None,
                  rows_per_chunk=None, max_iters: int = 64, heads=None, round_out: bool = True):
    """One attention layer's chunked prefill ([QW] "Algorithm"): for each chunk
    [cs, e) of `chunk` queries over the keys [0, e), select the critical tokens
    per head from the chunk's last `last_q` queries with continuous positions,
    optionally refine the budgets, then attend the chunk's rows with DCA
    positions (dca = (C, W)) or continuous ones.

    q: (Hq, N, d), k/v: (Hkv, N, d) float64 (bf16 values, pre-RoPE).
    kv_budget / ks_budget: one int for every head, or a sequence with one budget
    per head (calibrated budgets, used with tau None).
    rows_per_chunk: None (every row) or a function (cs, e) -> absolute rows to
    evaluate. round_out: False keeps the outputs in float64 (before the final
    bf16 rounding). Returns a list with one dict per chunk."""
    hq, n, d = q.shape
    hkv = k.shape[0]
    g = hq // hkv
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    heads = range(hq) if heads is None else heads
    res = []
    for cs in range(0, n, chunk):
        e = min(cs + chunk, n)
        nr = min(last_q, e - cs)
        est_rows = np.arange(e - nr, e)
        rows = np.arange(cs, e) if rows_per_chunk is None else np.asarray(rows_per_chunk(cs, e))
        per = {}
        for h in heads:
            kh, vh = k[h // g], v[h // g]
            kvb = int(kv_budget) if np.isscalar(kv_budget) else int(kv_budget[h])
            ksb = int(ks_budget) if np.isscalar(ks_budget) else int(ks_budget[h])
            lse_e, vert, slash, a = estimate(q[h, e - nr : e], kh, e, base, scale)
            if tau is None:
                kv, ks = min(kvb, e), min(ksb, e)
                V, S = select(vert, slash, kv, ks)
                rc = recall(a, est_rows, membership(e, V), membership(e, S))
                trace = [(kv, ks, rc)]
            else:
                kv, ks, V, S, rc, trace = refine(a, est_rows, vert, slash, kvb, ksb, tau, max_iters)
            o, lse = attention_rows(q[h, rows], rows, kh, vh, e, membership(e, V), membership(e, S),
                                    base, scale, dca, round_out=round_out)
            per[h] = dict(lse_est=lse_e, vert=vert, slash=slash, kv=kv, ks=ks, V=V, S=S,
                          recall=rc, trace=trace, rows=rows, out=o, lse=lse)
        res.append(dict(cs=cs, e=e, heads=per))
    return res
