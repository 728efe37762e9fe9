"""Full-size parity: the eight workloads at their real sizes, run through the
same chunk loop the benchmark times, checked against the oracle.

Sampling. Workloads 1-6: every chunk and every head (the complete vertical and
slash index sets of every (chunk, head) pair), and 512 query rows per head,
uniform without replacement over the sequence from numpy default_rng(seed +
1000), sorted, the same rows for every head (all 4096 rows at workload 1).
Workloads 7, 8 and 9 (1M-token variants beyond the five configurations) check a
fixed subset of chunks and heads. The oracle side runs in one process per KV
head group (tests/fullsize_oracle.py), fed chunk by chunk while the GPU loop
continues.
"""
import multiprocessing as mp
import os
import queue
import time

import numpy as np
import pytest
import torch

import sparse_attention_estimate_b200 as vsb
from sparse_attention_estimate_b200 import build as vsbuild
from tests import fullsize_oracle
from workloads import WORKLOADS, generate_head, structure

pytestmark = pytest.mark.gpu

# workload -> (chunks to check or None for all, heads to check or None for all, rows per head)
PLAN = {
    1: (None, None, 4096),
    2: (None, None, 512),
    3: (None, None, 512),
    4: (None, None, 512),
    5: (None, None, 512),
    6: (None, None, 512),
    7: ([0, 15, 31], [0, 21, 39], 64),
    8: ([31], [0, 17], 32),
    9: ([0, 8, 31], [0, 21, 39], 64),
}


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    vsbuild.build()
    vsb.load_library()


def sampled_rows(w, chunks, nrows):
    """The checked query rows: uniform without replacement over the checked chunks'
    rows (the whole sequence when every chunk is checked), sorted."""
    pool = np.concatenate([np.arange(*w.chunk_bounds(c)) for c in chunks])
    if nrows >= len(pool):
        return pool
    rng = np.random.default_rng(w.seed + 1000)
    return np.sort(rng.choice(pool, nrows, replace=False))


def _cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


@pytest.mark.parametrize("cfg", sorted(PLAN))
def test_fullsize_workload(cfg):
    w = WORKLOADS[cfg]
    chunks_sel, heads_sel, nrows = PLAN[cfg]
    chunks = list(range(w.n_chunks)) if chunks_sel is None else chunks_sel
    heads = list(range(w.hq)) if heads_sel is None else heads_sel
    rows = sampled_rows(w, chunks, nrows)
    est_rows = np.concatenate([np.arange(e - min(w.last_q, e - cs), e)
                               for cs, e in (w.chunk_bounds(c) for c in chunks)])
    groups = sorted({h // w.group for h in heads})

    # oracle workers, one per KV-head group (spawned: no CUDA state is inherited)
    ctx_mp = mp.get_context("spawn")
    threads = max(1, _cores() // max(1, len(groups)))
    saved = {k: os.environ.get(k) for k in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")}
    for k in saved:
        os.environ[k] = str(threads)
    result_q = ctx_mp.Queue()
    tasks, procs = {}, {}
    try:
        for hk in groups:
            tasks[hk] = ctx_mp.Queue(maxsize=3)
            gh = [h for h in heads if h // w.group == hk]
            procs[hk] = ctx_mp.Process(target=fullsize_oracle.worker_main,
                                       args=(w, hk, gh, rows, est_rows, tasks[hk], result_q), daemon=True)
            procs[hk].start()
    finally:
        for k, v in saved.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v

    failures = []
    try:
        _run_gpu_and_feed(w, chunks, heads, rows, groups, tasks, procs, result_q, failures)
    finally:
        for p in procs.values():
            p.join(timeout=5)
            if p.is_alive():
                p.kill()
    assert not failures, "\n".join(failures[:40]) + f"\n({len(failures)} failures)"


def _collect(result_q, pending, failures, block, deadline):
    while pending:
        try:
            c, hk, fails = result_q.get(timeout=5.0 if block else 0.0)
        except queue.Empty:
            if not block:
                return
            if time.time() > deadline:
                failures.append(f"oracle workers timed out with {len(pending)} results pending")
                return
            continue
        if c == "error":
            failures.extend(fails)
            pending.clear()
            return
        if c == "ready":
            continue
        pending.discard((c, hk))
        failures.extend(fails)


def _run_gpu_and_feed(w, chunks, heads, rows, groups, tasks, procs, result_q, failures):
    """The chunk loop of bench.py (estimate -> select/refine -> sparse prefill per
    chunk) on device-resident inputs; after each checked chunk its results go to
    the workers of the checked groups."""
    st = structure(w)
    dev = "cuda"
    q = torch.empty(w.hq, w.seq_len, 128, dtype=torch.bfloat16, device=dev)
    k = torch.empty(w.hkv, w.seq_len, 128, dtype=torch.bfloat16, device=dev)
    v = torch.empty(w.hkv, w.seq_len, 128, dtype=torch.bfloat16, device=dev)
    for name, t, nh in (("q", q, w.hq), ("k", k, w.hkv), ("v", v, w.hkv)):
        for h in range(nh):
            t[h].copy_(generate_head(w, name, h, st=st))
    cfg = vsb.Config(hq=w.hq, hkv=w.hkv, rope_base=w.rope_base, last_q=w.last_q, dca_chunk=w.dca_chunk,
                     dca_window=w.dca_window, softmax_scale=w.softmax_scale)
    ctx = vsb.Context(cfg, max_seq=w.seq_len, max_chunk=min(w.chunk, w.seq_len))
    out = torch.empty_like(q)
    lse_o = torch.empty(w.hq, w.seq_len, dtype=torch.float32, device=dev)
    rows_t = torch.as_tensor(rows, device=dev)
    pending = {(c, hk) for c in chunks for hk in groups}
    deadline = time.time() + 3600
    for c in range(w.n_chunks):
        cs, e = w.chunk_bounds(c)
        vert, slash, lse = ctx.estimate(q, cs, k, e, full=True)
        kv = torch.full((w.hq,), w.kv_budget, dtype=torch.int32, device=dev)
        ks = torch.full((w.hq,), w.ks_budget, dtype=torch.int32, device=dev)
        recall = None
        if w.refine_tau is None:
            sets = ctx.select(vert, slash, e, kv, ks)
        else:
            sets, recall = ctx.refine(q, cs, k, e, vert, slash, lse, w.refine_tau, kv, ks, full=True)
        ctx.sparse_prefill(q, cs, e, k, v, sets, out=out, lse=lse_o, full=True)
        if c in chunks:
            sel = (rows >= cs) & (rows < e)
            rt = rows_t[torch.as_tensor(sel, device=dev)]
            v_idx, v_cnt, s_off, s_cnt = [t.cpu().numpy() for t in sets]
            vh, sh = vert.cpu().numpy(), slash.cpu().numpy()
            kvh, ksh = kv.cpu().numpy(), ks.cpu().numpy()
            rch = None if recall is None else recall.cpu().numpy()
            oh = out[:, rt].float().cpu().numpy()
            lh = lse_o[:, rt].cpu().numpy()
            for hk in groups:
                per = {}
                for h in heads:
                    if h // w.group != hk:
                        continue
                    per[h] = dict(vert=vh[h], slash=sh[h], kv=int(kvh[h]), ks=int(ksh[h]),
                                  recall=None if rch is None else float(rch[h]),
                                  V=v_idx[h, : v_cnt[h]].astype(np.int64), S=s_off[h, : s_cnt[h]].astype(np.int64),
                                  out=oh[h], lse=lh[h])
                while True:  # bounded queues: wait for slow workers, reporting what they found meanwhile
                    try:
                        tasks[hk].put((c, cs, e, per), timeout=5.0)
                        break
                    except queue.Full:
                        _collect(result_q, pending, failures, False, deadline)
                        if not procs[hk].is_alive():
                            failures.append(f"oracle worker of KV group {hk} died")
                            return
            del v_idx, s_off, vh, sh
        _collect(result_q, pending, failures, False, deadline)
        del vert, slash, lse, sets
    torch.cuda.synchronize()
    assert ctx.status() == vsb.VS_OK
    for hk in groups:
        tasks[hk].put(None)
    _collect(result_q, pending, failures, True, deadline)
