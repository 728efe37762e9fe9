"""Full-size parity: the eight workloads at their real sizes, run through the
same chunk loop the benchmark times, checked against the oracle on sampled
query rows, on the complete index sets of sampled (chunk, head) pairs, and on
properties that hold at any size.

Sampling (fixed seeds): workloads 1, 2 and 6 check every head; 3-5, 7, 8 check a fixed
subset of chunks and heads (the oracle's fp64 estimation of one (chunk, head)
at e = 1M costs seconds). Rows: uniform without replacement from
numpy default_rng(seed + 1000), sorted, the same rows for every checked head.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle.vs_oracle as vo
import sparse_attention_estimate_b200 as vsb
from sparse_attention_estimate_b200 import build as vsbuild
from tests.gpu_common import TAU_SLACK, assert_near_tie_equal, assert_outputs_close, f64, sets_to_lists
from workloads import WORKLOADS, generate_head, structure

pytestmark = pytest.mark.gpu

# workload -> (chunks to check, heads to check, rows per checked (chunk, head))
PLAN = {
    1: (None, None, 4096),
    2: (None, None, 64),
    3: ([0, 3], [0, 13, 27], 32),
    4: ([0, 3, 7], [0, 21, 39], 32),
    5: ([0, 9, 31], [0, 39], 16),
    6: (None, None, 64),
    7: ([0, 31], [0, 39], 16),
    8: ([31], [0, 17], 16),
}


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    vsbuild.build()
    vsb.load_library()


def _run_gpu(w, check_chunks):
    """The chunk loop of bench.py (estimate -> select/refine -> sparse prefill per
    chunk) on device-resident inputs; returns host copies of what the checks of
    the chunks in `check_chunks` need, and the whole output."""
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
    res = {}
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
        if c in check_chunks:
            res[c] = dict(cs=cs, e=e, vert=vert.cpu(), slash=slash.cpu(), kv=kv.cpu().numpy(),
                          ks=ks.cpu().numpy(), recall=None if recall is None else recall.cpu().numpy(),
                          sets=sets_to_lists(sets), lse=lse_o[:, cs:e].cpu())
        del vert, slash, lse, sets
    torch.cuda.synchronize()
    assert ctx.status() == vsb.VS_OK
    return res, out, st


@pytest.mark.parametrize("cfg", sorted(PLAN))
def test_fullsize_workload(cfg):
    w = WORKLOADS[cfg]
    chunks_sel, heads_sel, nrows = PLAN[cfg]
    chunks = list(range(w.n_chunks)) if chunks_sel is None else chunks_sel
    res, out, st = _run_gpu(w, set(chunks))
    scale = w.softmax_scale
    dca = (w.dca_chunk, w.dca_window) if w.dca_chunk else None
    heads = range(w.hq) if heads_sel is None else heads_sel
    rng = np.random.default_rng(w.seed + 1000)
    kcache = {}
    for c in chunks:
        r = res[c]
        cs, e = r["cs"], r["e"]
        assert cs == c * w.chunk
        nr = min(w.last_q, e - cs)
        est_rows = np.arange(e - nr, e)
        rows = np.arange(cs, e) if nrows >= e - cs else np.sort(rng.choice(np.arange(cs, e), nrows, replace=False))
        vert, slash = f64(r["vert"]), f64(r["slash"])
        V, S = r["sets"]
        # properties at any size: probability mass per estimation row
        assert np.allclose(vert.sum(1), nr, rtol=1e-4) and np.allclose(slash.sum(1), nr, rtol=1e-4)
        for h in heads:
            hk = h // w.group
            if hk not in kcache:
                kcache.clear()
                kcache[hk] = (generate_head(w, "k", hk, st=st).float().double().numpy(),
                              generate_head(w, "v", hk, st=st).float().double().numpy())
            kf, vf = kcache[hk]
            qh = generate_head(w, "q", h, rows=torch.from_numpy(np.concatenate([est_rows, rows])), st=st)
            qh = qh.float().double().numpy()
            q_est, q_rows = qh[:nr], qh[nr:]
            # the GPU's sets are exactly the selection of its own scores at its final budgets
            kv, ks = int(r["kv"][h]), int(r["ks"][h])
            ov, osl = vo.select(vert[h], slash[h], kv, ks)
            assert np.array_equal(V[h], ov) and np.array_equal(S[h], osl), (cfg, c, h)
            # estimation and selection against the oracle's fp64 scores (near-ties allowed)
            _, overt, oslash, a = vo.estimate(q_est, kf, e, w.rope_base, scale)
            tol = 2e-5 * overt.max() + 1e-4 * np.abs(overt)
            assert np.all(np.abs(vert[h] - overt) <= tol), (cfg, c, h)
            if w.refine_tau is None:
                okv, oks = min(w.kv_budget, e), min(w.ks_budget, e)
            else:
                okv, oks, _, _, orc, trace = vo.refine(a, est_rows, overt, oslash, w.kv_budget, w.ks_budget,
                                                       w.refine_tau)
                if (okv, oks) != (kv, ks):
                    assert any(abs(x - w.refine_tau) < TAU_SLACK for _, _, x in trace), (cfg, c, h, trace, kv)
                    okv, oks = kv, ks
                else:
                    assert abs(r["recall"][h] - orc) < 1e-4, (cfg, c, h, r["recall"][h], orc)
            oV, oS = vo.select(overt, oslash, okv, oks)
            assert_near_tie_equal(V[h], oV, overt, okv)
            sl = oslash.copy()
            sl[0] = np.inf
            assert_near_tie_equal(S[h], oS, sl, oks)
            # attention of the sampled rows with the GPU's sets
            oo, ol = vo.attention_rows(q_rows, rows, kf, vf, e, vo.membership(e, V[h]), vo.membership(e, S[h]),
                                       w.rope_base, scale, dca)
            got = f64(out[h][torch.as_tensor(rows, device=out.device)])
            assert_outputs_close(got, oo, f"cfg{cfg} chunk {c} head {h}", w=w)
            assert np.allclose(f64(r["lse"][h, rows - cs]), ol, rtol=0, atol=2e-3), (cfg, c, h)
