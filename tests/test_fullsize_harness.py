"""The checks of the full-size parity harness (tests/fullsize_oracle.py), on CPU:
results the oracle itself produces must pass every check, and results with one
planted fault (a wrong set member, a refinement level too far, a perturbed
output or score) must each be reported. The spawned-worker plumbing runs once on
a small workload."""
import multiprocessing as mp

import numpy as np
import pytest

import oracle.vs_oracle as vo
from tests import fullsize_oracle as fo
from workloads import generate_layer, small_workload

W = small_workload(2, seq_len=900, chunk=384, hq=4, hkv=2, n_planted=8, kv_budget=20, ks_budget=30,
                   refine_tau=0.9)


def _oracle_results(w, c, h, rows):
    """What a correct GPU would report for (chunk c, head h), from the oracle."""
    lay = generate_layer(w)
    q, k, v = (lay[x].float().double().numpy() for x in ("q", "k", "v"))
    cs, e = w.chunk_bounds(c)
    nr = min(w.last_q, e - cs)
    est = np.arange(e - nr, e)
    hk = h // w.group
    _, vert, slash, a = vo.estimate(q[h, e - nr : e], k[hk], e, w.rope_base, w.softmax_scale)
    kv, ks, V, S, rc, _ = vo.refine(a, est, vert, slash, w.kv_budget, w.ks_budget, w.refine_tau)
    out, lse = vo.attention_rows(q[h, rows], rows, k[hk], v[hk], e, vo.membership(e, V), vo.membership(e, S),
                                 w.rope_base, w.softmax_scale)
    gpu = dict(vert=vert.astype(np.float32), slash=slash.astype(np.float32), kv=kv, ks=ks, recall=rc,
               V=V, S=S, out=out, lse=lse)
    k_rot = fo.rope_blocked(vo, k[hk], np.arange(w.seq_len), w.rope_base)
    return gpu, dict(q_est=q[h, e - nr : e], q_rows=q[h, rows], k_rot=k_rot, v=v[hk], cs=cs, e=e), a, est


def _check(gpu, ctx, c, h, rows):
    return fo.check_head(vo, W, c, ctx["cs"], ctx["e"], h, gpu, ctx["q_est"], ctx["q_rows"], rows, ctx["k_rot"],
                         ctx["k_rot"], ctx["v"], None)


def test_oracle_results_pass_every_check():
    rows = np.array([770, 801, 899])
    for h in (0, 3):
        gpu, ctx, _, _ = _oracle_results(W, 2, h, rows)
        assert _check(gpu, ctx, 2, h, rows) == []


def test_planted_faults_are_reported():
    rows = np.array([770, 801, 899])
    gpu, ctx, a, est = _oracle_results(W, 2, 1, rows)
    e = ctx["e"]
    # a set member swapped for the strongest unselected column
    bad = dict(gpu)
    out_of_set = np.setdiff1d(np.arange(e), gpu["V"])
    worst_in = gpu["V"][np.argmin(gpu["vert"][gpu["V"]])]
    best_out = out_of_set[np.argmax(gpu["vert"][out_of_set])]
    bad["V"] = np.sort(np.append(np.setdiff1d(gpu["V"], [worst_in]), best_out))
    msgs = _check(bad, ctx, 2, 1, rows)
    assert any("vertical set is not the top" in m for m in msgs), msgs
    # one doubling level too far (sets and recall of that level, consistently)
    bad = dict(gpu)
    kv2, ks2 = min(2 * gpu["kv"], e), min(2 * gpu["ks"], e)
    if (kv2, ks2) != (gpu["kv"], gpu["ks"]):
        V2, S2 = vo.select(gpu["vert"].astype(np.float64), gpu["slash"].astype(np.float64), kv2, ks2)
        bad.update(kv=kv2, ks=ks2, V=V2, S=S2,
                   recall=vo.recall(a, est, vo.membership(e, V2), vo.membership(e, S2)))
        msgs = _check(bad, ctx, 2, 1, rows)
        assert any("already reaches tau" in m for m in msgs), msgs
    # an output element off by 0.05
    bad = dict(gpu)
    bad["out"] = gpu["out"].copy()
    bad["out"][1, 7] += 0.05
    msgs = _check(bad, ctx, 2, 1, rows)
    assert any("outputs" in m for m in msgs), msgs
    # vertical scores off by 1 %
    bad = dict(gpu)
    bad["vert"] = gpu["vert"] * np.float32(1.01)
    msgs = _check(bad, ctx, 2, 1, rows)
    assert any("vert off" in m for m in msgs), msgs


def test_topk_and_near_tie_helpers():
    s = np.array([5.0, 3.0, 3.0, 3.0, 1.0, 0.0])
    assert fo.is_exact_topk(s, np.array([0, 1, 2]), 3)
    assert not fo.is_exact_topk(s, np.array([0, 1, 3]), 3)  # tie broken by the higher index
    assert not fo.is_exact_topk(s, np.array([0, 1]), 3)
    assert fo.is_exact_topk(s, np.arange(6), 9)
    assert fo.near_tie_violations(np.array([0, 1, 3]), s, 3, 3.0) == []  # differs only in a tie
    assert fo.near_tie_violations(np.array([0, 1, 4]), s, 3, 3.0) == [4]  # 1.0 is no near tie of 3.0
    assert fo.near_tie_violations(np.array([1, 2, 3]), s, 3, 3.0) == [0]  # 5.0 left out


def test_worker_process_reports_results():
    """The spawned worker regenerates the inputs, receives one chunk and reports."""
    w = W
    c, h = 1, 2
    cs, e = w.chunk_bounds(c)
    rows = np.array([cs + 5, e - 1])
    gpu, _, _, _ = _oracle_results(w, c, h, rows)
    est = np.arange(e - min(w.last_q, e - cs), e)
    ctx = mp.get_context("spawn")
    task_q, result_q = ctx.Queue(), ctx.Queue()
    p = ctx.Process(target=fo.worker_main, args=(w, h // w.group, [h], rows, est, task_q, result_q), daemon=True)
    p.start()
    try:
        task_q.put((c, cs, e, {h: gpu}))
        task_q.put(None)
        got = [result_q.get(timeout=120) for _ in range(2)]
    finally:
        p.join(timeout=30)
        if p.is_alive():
            p.kill()
    assert got[0][0] == "ready"
    assert got[1] == (c, h // w.group, []), got[1]
