"""Oracle side of the full-size parity tests (TEST INFRASTRUCTURE; imports oracle/).

The GPU test process runs the chunk loop and hands each chunk's results, split by
KV-head group, to one worker process per group (multiprocessing, `spawn`). A
worker regenerates its group's inputs from the seeded generator, rotates its
keys once (the oracle's rope over blocks of rows: rows are independent, so the
result is the same array), and checks every (chunk, head) it receives against
the float64 oracle:

  mass       vertical and slash sums of every estimation row add up to 1
  selection  the GPU's sets are exactly the top-k of the GPU's own scores at its
             final budgets (index-exact; ties by ascending index)
  estimate   vertical and slash scores within 2e-5 of the largest score plus
             1e-4 relative of the oracle's
  refinement the GPU's final budgets are the first doubling level whose oracle
             recall reaches tau (or saturation): recall is non-decreasing over
             the nested levels, so the oracle's level-by-level loop stops at the
             GPU's level t exactly when recall(t) >= tau (or t saturates) and
             recall(t - 1) < tau; decisions within TAU_SLACK of tau go either way
  near ties  the GPU's sets differ from the oracle's selection on the oracle's
             scores (same budgets) only by elements within 1e-4 relative of the
             oracle's k-th score
  attention  sampled query rows of the chunk, with the GPU's sets, against the
             oracle's attention (outputs and lse)

Workers report failures as strings; the test asserts there are none.
"""
from __future__ import annotations

import math
import os
import traceback

import numpy as np

NEAR_TIE_REL = 1e-4
TAU_SLACK = 1e-5
OUT_MAX_ABS = 2e-2
OUT_MEAN_ABS = 2e-3
ROPE_BLOCK = 8192


def rope_blocked(vo, x: np.ndarray, pos: np.ndarray, base: float) -> np.ndarray:
    """vo.rope over blocks of rows (each row is rotated on its own)."""
    out = np.empty_like(x)
    for r0 in range(0, x.shape[0], ROPE_BLOCK):
        out[r0 : r0 + ROPE_BLOCK] = vo.rope(x[r0 : r0 + ROPE_BLOCK], pos[r0 : r0 + ROPE_BLOCK], base)
    return out


def is_exact_topk(score: np.ndarray, sel: np.ndarray, k: int) -> bool:
    """True when `sel` (ascending indices) is the top-k of `score` ranked by (score
    descending, index ascending): k elements, none of the others ranked above any
    selected one."""
    n = score.shape[0]
    k = min(int(k), n)
    if sel.shape[0] != k or (k and (np.any(np.diff(sel) <= 0) or sel[0] < 0 or sel[-1] >= n)):
        return False
    if k == 0 or k == n:
        return True
    inm = np.zeros(n, dtype=bool)
    inm[sel] = True
    lo = score[inm].min()       # weakest selected score
    hi = score[~inm].max()      # strongest unselected score
    if lo > hi:
        return True
    if lo < hi:
        return False
    # equal scores at the boundary: selected ones must have the lower indices
    return int(np.flatnonzero(inm & (score == lo)).max()) < int(np.flatnonzero(~inm & (score == hi)).min())


def near_tie_violations(got: np.ndarray, score: np.ndarray, k: int, kth: float) -> list:
    """Elements by which `got` (a k-set) differs from the exact top-k of `score`
    that are not within NEAR_TIE_REL of the k-th score `kth`: selected elements
    clearly below it and unselected ones clearly above it."""
    n = score.shape[0]
    tol = NEAR_TIE_REL * abs(kth) + 1e-30 if np.isfinite(kth) else 0.0
    inm = np.zeros(n, dtype=bool)
    inm[got] = True
    bad_in = np.flatnonzero(inm & (score < kth - tol))
    bad_out = np.flatnonzero(~inm & (score > kth + tol))
    return [int(x) for x in bad_in[:5]] + [int(x) for x in bad_out[:5]]


def bf16_half_ulp(x: np.ndarray) -> np.ndarray:
    a = np.abs(x)
    ex = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return np.where(a > 0, np.exp2(ex - 8), 0.0)


def output_violation(vo, got: np.ndarray, exact: np.ndarray, peaked: bool):
    """None when the outputs agree (the bounds of tests/gpu_common.py), else a message."""
    if peaked:
        d = np.abs(got - exact)
        hu = bf16_half_ulp(exact)
        if np.any(d > OUT_MAX_ABS + hu):
            return f"max excess {np.max(d - hu):.3e}"
        if d.mean() > OUT_MEAN_ABS + hu.mean():
            return f"mean {d.mean():.3e}"
        return None
    d = np.abs(got - vo.bf16_rne(exact))
    if d.max() > OUT_MAX_ABS:
        return f"max abs {d.max():.3e}"
    if d.mean() > OUT_MEAN_ABS:
        return f"mean abs {d.mean():.3e}"
    return None


def level_budgets(kv0: int, ks0: int, e: int, t: int):
    """Budgets of doubling level t (both capped at e)."""
    return min(kv0 << t, e), min(ks0 << t, e)


def check_head(vo, w, c, cs, e, h, gpu, q_est, q_rows, rows, k_rot, k_attn, v, dca) -> list:
    """Every check of one (chunk, head); returns failure messages."""
    fails = []
    where = f"cfg {w.name} chunk {c} head {h}"
    nr = q_est.shape[0]
    est_rows = np.arange(e - nr, e)
    vert = gpu["vert"].astype(np.float64)
    slash = gpu["slash"].astype(np.float64)
    V, S = gpu["V"], gpu["S"]
    kv, ks = int(gpu["kv"]), int(gpu["ks"])
    # mass of the estimation rows
    if not (abs(vert.sum() - nr) <= 1e-4 * nr and abs(slash.sum() - nr) <= 1e-4 * nr):
        fails.append(f"{where}: mass {vert.sum():.6f} {slash.sum():.6f} vs {nr}")
    # the GPU's sets are the exact selection of its own scores
    if not is_exact_topk(vert, V, kv):
        fails.append(f"{where}: vertical set is not the top-{kv} of the GPU scores")
    if not is_exact_topk(vo.slash_scores(slash), S, ks):
        fails.append(f"{where}: slash set is not the top-{ks} of the GPU scores")
    # the oracle's estimate
    _, overt, oslash, a = vo.estimate(q_est, None, e, w.rope_base, w.softmax_scale, k_rot=k_rot)
    for name, got, want in (("vert", vert, overt), ("slash", slash, oslash)):
        tol = 2e-5 * want.max() + 1e-4 * np.abs(want)
        if np.any(np.abs(got - want) > tol):
            fails.append(f"{where}: {name} off by {np.max(np.abs(got - want) / want.max()):.3e} of the max")
    orders = vo.select_orders(overt, oslash)
    # refinement decision
    if w.refine_tau is not None:
        tau = w.refine_tau
        t = 0
        while level_budgets(w.kv_budget, w.ks_budget, e, t) != (kv, ks):
            t += 1
            if t > 40:
                fails.append(f"{where}: budgets ({kv}, {ks}) are no doubling level of the base budgets")
                break
        if t <= 40:
            def rc(level):
                a_v, a_s = level_budgets(w.kv_budget, w.ks_budget, e, level)
                oV, oS = vo.select(overt, oslash, a_v, a_s, orders)
                return vo.recall(a, est_rows, vo.membership(e, oV), vo.membership(e, oS))
            r_t = rc(t)
            saturated = kv >= e and ks >= e
            if r_t < tau and not saturated and t < 19 and abs(r_t - tau) >= TAU_SLACK:
                fails.append(f"{where}: stopped at level {t} with oracle recall {r_t:.6f} < tau")
            if t > 0:
                r_p = rc(t - 1)
                if r_p >= tau and abs(r_p - tau) >= TAU_SLACK:
                    fails.append(f"{where}: level {t - 1} already reaches tau (oracle recall {r_p:.6f})")
            if gpu.get("recall") is not None and abs(float(gpu["recall"]) - r_t) >= 1e-4 and \
                    abs(r_t - tau) >= TAU_SLACK:
                fails.append(f"{where}: recall {float(gpu['recall']):.6f} vs oracle {r_t:.6f}")
    # the GPU's sets against the oracle's selection at the same budgets (near ties allowed)
    ov, osl = orders
    for name, got, score, k, order in (("vertical", V, overt, kv, ov),
                                       ("slash", S, vo.slash_scores(oslash), ks, osl)):
        kth = vo.kth_score(score, k, order=order)
        bad = near_tie_violations(got, score, k, kth)
        if bad:
            fails.append(f"{where}: {name} set differs from the oracle's beyond near ties at {bad}")
    del a
    # attention of the sampled rows with the GPU's sets
    if len(rows):
        oo, ol = vo.attention_rows(q_rows, rows, None, v, e, vo.membership(e, V), vo.membership(e, S),
                                   w.rope_base, w.softmax_scale, dca, k_rot=k_attn, round_out=False)
        msg = output_violation(vo, gpu["out"].astype(np.float64), oo, w.q_scale != 1.0)
        if msg:
            fails.append(f"{where}: outputs {msg}")
        dl = np.abs(gpu["lse"].astype(np.float64) - ol)
        if np.any(dl > 2e-3):
            fails.append(f"{where}: lse off by {dl.max():.3e}")
    return fails


def worker_main(w, hk: int, heads: list, rows_all: np.ndarray, est_rows_all: np.ndarray,
                task_q, result_q) -> None:
    """One KV-head group: regenerate inputs, rotate keys once, then check the chunks
    that arrive on task_q (None ends the loop). Puts (chunk, failures) on result_q."""
    try:
        import oracle.vs_oracle as vo
        import torch
        from workloads import generate_head, structure

        torch.set_num_threads(1)
        st = structure(w)
        dca = (w.dca_chunk, w.dca_window) if w.dca_chunk else None
        kf = generate_head(w, "k", hk, st=st).float().double().numpy()
        v = generate_head(w, "v", hk, st=st).float().double().numpy()
        n = w.seq_len
        k_rot = rope_blocked(vo, kf, np.arange(n), w.rope_base)
        k_attn = k_rot if dca is None else rope_blocked(vo, kf, vo.key_positions(n, dca), w.rope_base)
        del kf
        need = np.union1d(rows_all, est_rows_all)
        qcache = {}
        for h in heads:
            qh = generate_head(w, "q", h, rows=torch.from_numpy(need), st=st).float().double().numpy()
            qcache[h] = dict(zip(need.tolist(), qh))
        result_q.put(("ready", hk, []))
        while True:
            task = task_q.get()
            if task is None:
                break
            c, cs, e, per_head = task
            nr = min(w.last_q, e - cs)
            est = np.arange(e - nr, e)
            rows = rows_all[(rows_all >= cs) & (rows_all < e)]
            fails = []
            for h, gpu in per_head.items():
                q_est = np.stack([qcache[h][int(i)] for i in est])
                q_rows = np.stack([qcache[h][int(i)] for i in rows]) if len(rows) else np.zeros((0, 128))
                try:
                    fails += check_head(vo, w, c, cs, e, h, gpu, q_est, q_rows, rows, k_rot, k_attn, v, dca)
                except Exception:
                    fails.append(f"cfg {w.name} chunk {c} head {h}: {traceback.format_exc(limit=3)}")
            result_q.put((c, hk, fails))
    except Exception:
        result_q.put(("error", hk, [traceback.format_exc()]))
