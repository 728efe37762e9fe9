"""Parity of every library call with the CPU oracle, on small seeded workloads
that span several 128-row tiles / 128-key blocks and end in ragged tails."""
import ctypes

import numpy as np
import pytest
import torch

import oracle.vs_oracle as vo
import sparse_attention_estimate_b200 as vsb
from sparse_attention_estimate_b200 import build as vsbuild
from tests.gpu_common import (OUT_MAX_ABS, TAU_SLACK, assert_near_tie_equal, assert_outputs_close, f64,
                              layer_inputs, lists_to_sets, make_ctx, scale_of, sets_to_lists)
from workloads import generate_head, generate_layer, small_workload, structure

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    vsbuild.build()
    vsb.load_library()


# (workload, dca (C, W) or None): group sizes 2, 7 and 5; ragged tails; DCA with all three classes
CASES = {
    "g2_two_chunks": (small_workload(2, seq_len=1000, chunk=512, hq=4, hkv=2, n_planted=8, kv_budget=40,
                                     ks_budget=60, refine_tau=0.9), None),
    "g7_one_chunk": (small_workload(2, seq_len=700, chunk=700, hq=7, hkv=1, n_planted=8, kv_budget=30,
                                    ks_budget=50, refine_tau=0.9), None),
    "g5_dca": (small_workload(5, seq_len=1400, chunk=512, hq=5, hkv=1, n_planted=16, kv_budget=64,
                              ks_budget=96, refine_tau=0.9), (512, 128)),
    # MHA (group 1: half-empty estimation tile); the last chunk holds a single row
    "g1_tail1": (small_workload(2, seq_len=641, chunk=640, hq=2, hkv=2, n_planted=4, kv_budget=20,
                                ks_budget=30, refine_tau=0.9), None),
    # sparse regime (base logits with std 4) and the YaRN temperature (s = 1400 / 512)
    "g4_peaked": (small_workload(6, seq_len=1100, chunk=512, hq=4, hkv=1, n_planted=8, kv_budget=40,
                                 ks_budget=60, refine_tau=0.9), None),
    "g5_dca_yarn": (small_workload(8, seq_len=1400, chunk=512, hq=5, hkv=1, n_planted=16, kv_budget=64,
                                   ks_budget=96, refine_tau=0.9, yarn_train_len=512), (512, 128)),
}


@pytest.fixture(scope="module", params=list(CASES))
def case(request):
    w, dca = CASES[request.param]
    dev, cpu = layer_inputs(w)
    ctx = make_ctx(w, dca=dca)
    return request.param, w, dca, dev, cpu, ctx


def _chunks(w):
    return [w.chunk_bounds(c) for c in range(w.n_chunks)]


def test_dca_remap_matches_oracle(case):
    name, w, dca, dev, cpu, ctx = case
    pk, pqi, pqs, pqx = [t.cpu().numpy() for t in ctx.dca_remap(0, w.seq_len)]
    t = np.arange(w.seq_len)
    if dca is None:
        for a in (pk, pqi, pqs, pqx):
            assert np.array_equal(a, t)
        return
    C, W = dca
    assert np.array_equal(pk, t % (C - W))
    for cls, arr in enumerate((pqi, pqs, pqx)):
        assert np.array_equal(arr, [vo.dca_q_position(int(i), cls, C, W) for i in t])


def test_estimate_matches_oracle(case):
    name, w, dca, dev, cpu, ctx = case
    scale = scale_of(w)
    for cs, e in _chunks(w):
        qc = dev["q"][:, cs:e].contiguous()
        vert, slash, lse = ctx.estimate(qc, cs, dev["k"], e)
        vert, slash, lse = f64(vert), f64(slash), f64(lse)
        nr = min(w.last_q, e - cs)
        for h in range(w.hq):
            ol, ov, osl, _ = vo.estimate(cpu["q"][h, e - nr : e], cpu["k"][h // w.group], e, w.rope_base, scale)
            assert np.allclose(lse[h, :nr], ol, rtol=0, atol=2e-5), (name, cs, h)
            assert np.all(np.isneginf(lse[h, nr:]))
            for got, want in ((vert[h], ov), (slash[h], osl)):
                tol = 2e-5 * want.max() + 1e-4 * np.abs(want)
                assert np.all(np.abs(got - want) <= tol), (name, cs, h, np.max(np.abs(got - want) / want.max()))
            assert abs(vert[h].sum() - nr) < 1e-3 and abs(slash[h].sum() - nr) < 1e-3


def test_estimate_is_deterministic(case):
    name, w, dca, dev, cpu, ctx = case
    cs, e = _chunks(w)[-1]
    qc = dev["q"][:, cs:e].contiguous()
    a = [t.clone() for t in ctx.estimate(qc, cs, dev["k"], e)]
    b = ctx.estimate(qc, cs, dev["k"], e)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_select_exact_on_identical_scores(case):
    """Given the same scores, selection is index-exact (bit-exact integer work)."""
    name, w, dca, dev, cpu, ctx = case
    for cs, e in _chunks(w):
        qc = dev["q"][:, cs:e].contiguous()
        vert, slash, _ = ctx.estimate(qc, cs, dev["k"], e)
        for kv, ks in [(w.kv_budget, w.ks_budget), (1, 1), (e, e), (3 * e, 7), (0, 5)]:
            kvb = torch.full((w.hq,), kv, dtype=torch.int32, device="cuda")
            ksb = torch.full((w.hq,), ks, dtype=torch.int32, device="cuda")
            V, S = sets_to_lists(ctx.select(vert, slash, e, kvb, ksb))
            gv, gs = f64(vert), f64(slash)
            for h in range(w.hq):
                ov, osl = vo.select(gv[h], gs[h], kv, ks)
                assert np.array_equal(V[h], ov), (name, cs, kv, h)
                assert np.array_equal(S[h], osl), (name, cs, ks, h)
            assert ctx.status() == vsb.VS_OK


def test_select_with_ties():
    """Many exact ties: the index-ascending rule decides."""
    w = small_workload(2, seq_len=700, chunk=700, hq=4, hkv=2)
    ctx = make_ctx(w)
    g = torch.Generator().manual_seed(7)
    vert = (torch.randint(0, 6, (4, 700), generator=g).float() / 8).cuda()
    slash = (torch.randint(0, 3, (4, 700), generator=g).float() / 4).cuda()
    for kv, ks in [(10, 10), (333, 100), (699, 1)]:
        kvb = torch.full((4,), kv, dtype=torch.int32, device="cuda")
        ksb = torch.full((4,), ks, dtype=torch.int32, device="cuda")
        V, S = sets_to_lists(ctx.select(vert, slash, 700, kvb, ksb))
        for h in range(4):
            ov, osl = vo.select(f64(vert[h]), f64(slash[h]), kv, ks)
            assert np.array_equal(V[h], ov) and np.array_equal(S[h], osl)


def test_select_matches_oracle_scores_up_to_near_ties(case):
    name, w, dca, dev, cpu, ctx = case
    scale = scale_of(w)
    cs, e = _chunks(w)[-1]
    qc = dev["q"][:, cs:e].contiguous()
    vert, slash, _ = ctx.estimate(qc, cs, dev["k"], e)
    kvb = torch.full((w.hq,), w.kv_budget, dtype=torch.int32, device="cuda")
    ksb = torch.full((w.hq,), w.ks_budget, dtype=torch.int32, device="cuda")
    V, S = sets_to_lists(ctx.select(vert, slash, e, kvb, ksb))
    nr = min(w.last_q, e - cs)
    for h in range(w.hq):
        _, ov, osl, _ = vo.estimate(cpu["q"][h, e - nr : e], cpu["k"][h // w.group], e, w.rope_base, scale)
        oV, oS = vo.select(ov, osl, w.kv_budget, w.ks_budget)
        assert_near_tie_equal(V[h], oV, ov, w.kv_budget)
        sl = osl.copy()
        sl[0] = np.inf
        assert_near_tie_equal(S[h], oS, sl, w.ks_budget)


@pytest.mark.parametrize("tau", [0.3, 0.9, 0.999, 2.0])
def test_refine_matches_oracle(case, tau):
    name, w, dca, dev, cpu, ctx = case
    scale = scale_of(w)
    for cs, e in _chunks(w):
        qc = dev["q"][:, cs:e].contiguous()
        vert, slash, lse = ctx.estimate(qc, cs, dev["k"], e)
        kvb = torch.full((w.hq,), w.kv_budget, dtype=torch.int32, device="cuda")
        ksb = torch.full((w.hq,), w.ks_budget, dtype=torch.int32, device="cuda")
        sets, recall = ctx.refine(qc, cs, dev["k"], e, vert, slash, lse, tau, kvb, ksb)
        V, S = sets_to_lists(sets)
        kvb, ksb, recall = kvb.cpu().numpy(), ksb.cpu().numpy(), recall.cpu().numpy()
        gv, gs = f64(vert), f64(slash)
        nr = min(w.last_q, e - cs)
        rows = np.arange(e - nr, e)
        for h in range(w.hq):
            # the sets are the selection at the final budgets (on the same scores)
            ov, osl = vo.select(gv[h], gs[h], int(kvb[h]), int(ksb[h]))
            assert np.array_equal(V[h], ov) and np.array_equal(S[h], osl), (name, cs, h)
            # the decision follows the oracle's recall trace (fp64, its own estimate)
            _, ovv, oss, a = vo.estimate(cpu["q"][h, e - nr : e], cpu["k"][h // w.group], e, w.rope_base, scale)
            okv, oks, _, _, orc, trace = vo.refine(a, rows, ovv, oss, w.kv_budget, w.ks_budget, tau)
            if (okv, oks) != (int(kvb[h]), int(ksb[h])):
                # allowed only when a recall in the trace sits at tau
                assert any(abs(rc - tau) < TAU_SLACK for _, _, rc in trace), (name, cs, h, trace, kvb[h])
            else:
                assert abs(recall[h] - orc) < 1e-4, (name, cs, h, recall[h], orc)
        assert ctx.status() == vsb.VS_OK


@pytest.mark.parametrize("tau", [0.3, 0.9, 0.999])
def test_refine_recall_at_dca_positions(case, tau):
    """Refinement whose recall comes from the estimation rows' attention at DCA
    positions (selection still on continuous positions), against the oracle's
    refinement driven by estimate_probs_dca."""
    name, w, dca, dev, cpu, _ = case
    if dca is None:
        pytest.skip("no DCA")
    ctx = make_ctx(w, dca=dca, refine_dca_positions=True)
    scale = scale_of(w)
    for cs, e in _chunks(w):
        qc = dev["q"][:, cs:e].contiguous()
        vert, slash, lse = ctx.estimate(qc, cs, dev["k"], e)
        kvb = torch.full((w.hq,), w.kv_budget, dtype=torch.int32, device="cuda")
        ksb = torch.full((w.hq,), w.ks_budget, dtype=torch.int32, device="cuda")
        sets, recall = ctx.refine(qc, cs, dev["k"], e, vert, slash, lse, tau, kvb, ksb)
        assert ctx.status() == vsb.VS_OK
        V, S = sets_to_lists(sets)
        kvb, ksb, recall = kvb.cpu().numpy(), ksb.cpu().numpy(), recall.cpu().numpy()
        gv, gs = f64(vert), f64(slash)
        nr = min(w.last_q, e - cs)
        rows = np.arange(e - nr, e)
        for h in range(w.hq):
            ov, osl = vo.select(gv[h], gs[h], int(kvb[h]), int(ksb[h]))
            assert np.array_equal(V[h], ov) and np.array_equal(S[h], osl), (name, cs, h)
            qh, kh = cpu["q"][h, e - nr : e], cpu["k"][h // w.group]
            _, ovv, oss, _ = vo.estimate(qh, kh, e, w.rope_base, scale)
            _, a_dca = vo.estimate_probs_dca(qh, kh, e, w.rope_base, scale, dca)
            okv, oks, _, _, orc, trace = vo.refine(a_dca, rows, ovv, oss, w.kv_budget, w.ks_budget, tau)
            if (okv, oks) != (int(kvb[h]), int(ksb[h])):
                assert any(abs(rc - tau) < TAU_SLACK for _, _, rc in trace), (name, cs, h, trace, kvb[h])
            else:
                assert abs(recall[h] - orc) < 1e-4, (name, cs, h, recall[h], orc)


def _random_sets(rng, hq, e, pv, ps, force0=True):
    V, S = [], []
    for _ in range(hq):
        V.append(np.flatnonzero(rng.random(e) < pv).astype(np.int64))
        s = rng.random(e) < ps
        if force0:
            s[0] = True
        S.append(np.flatnonzero(s).astype(np.int64))
    return V, S


@pytest.mark.parametrize("density", ["sparse", "mixed", "full"])
def test_sparse_prefill_matches_oracle(case, density):
    name, w, dca, dev, cpu, ctx = case
    scale = scale_of(w)
    rng = np.random.default_rng(3)
    for cs, e in _chunks(w):
        pv, ps = {"sparse": (0.004, 0.004), "mixed": (0.3, 0.05), "full": (1.0, 1.0)}[density]
        V, S = _random_sets(rng, w.hq, e, pv, ps)
        sets = lists_to_sets(V, S, e, e)
        qc = dev["q"][:, cs:e].contiguous()
        out, lse = ctx.sparse_prefill(qc, cs, e, dev["k"], dev["v"], sets)
        assert ctx.status() == vsb.VS_OK
        out, lse = f64(out), f64(lse)
        rows = np.arange(cs, e)
        for h in range(w.hq):
            oo, ol = vo.attention_rows(cpu["q"][h, cs:e], rows, cpu["k"][h // w.group], cpu["v"][h // w.group], e,
                                       vo.membership(e, V[h]), vo.membership(e, S[h]), w.rope_base, scale, dca,
                                       round_out=False)
            assert_outputs_close(out[h], oo, f"{name} {density} cs={cs} h={h}", w=w)
            assert np.allclose(lse[h], ol, rtol=0, atol=2e-3), (name, density, cs, h, np.abs(lse[h] - ol).max())
        executed, useful = ctx.prefill_stats()
        assert executed > 0 and useful > 0


@pytest.mark.parametrize("density", ["full", "mixed"])
def test_sparse_prefill_with_large_jumps_of_the_row_max(density):
    """Keys whose logits dwarf everything before them, in the first and in the second
    64-key half of later 128-key blocks: the running row max of most query rows then
    rises by far more than 2^16 (and exp2 against the old max overflows), which sends
    the kernel's softmax through its redo-with-the-block's-own-max path and its O
    rescale. Checked against the oracle like every other prefill."""
    w = small_workload(2, seq_len=800, chunk=800, hq=2, hkv=1, n_planted=4)
    lay = generate_layer(w)
    spikes = [228, 276, 612, 670, 741]  # key offsets 100, 20, 100, 30, 101 inside their blocks
    lay["k"][0, spikes] = (lay["k"][0, spikes].float() * 40.0).to(torch.bfloat16)
    dev = {x: lay[x].cuda() for x in ("q", "k", "v")}
    cpu = {x: f64(lay[x]) for x in ("q", "k", "v")}
    ctx = make_ctx(w)
    e = w.seq_len
    if density == "full":
        V, S = [np.arange(e, dtype=np.int64)] * w.hq, [np.array([0], np.int64)] * w.hq
    else:
        V, S = _random_sets(np.random.default_rng(11), w.hq, e, 0.3, 0.05)
        V = [np.union1d(x, spikes).astype(np.int64) for x in V]
    out, lse = ctx.sparse_prefill(dev["q"], 0, e, dev["k"], dev["v"], lists_to_sets(V, S, e, e))
    assert ctx.status() == vsb.VS_OK
    out, lse = f64(out), f64(lse)
    rows = np.arange(e)
    for h in range(w.hq):
        oo, ol = vo.attention_rows(cpu["q"][h], rows, cpu["k"][0], cpu["v"][0], e, vo.membership(e, V[h]),
                                   vo.membership(e, S[h]), w.rope_base, scale_of(w), round_out=False)
        assert_outputs_close(out[h], oo, f"jumps {density} h={h}")
        assert np.allclose(lse[h], ol, rtol=0, atol=2e-3), (density, h, np.abs(lse[h] - ol).max())
    # the spikes do move the max: most rows past a spike attend mostly to it
    assert np.max(np.abs(ol)) > 50.0


def test_sparse_prefill_rows_without_keys_are_zero():
    w = small_workload(2, seq_len=640, chunk=640, hq=2, hkv=1)
    dev, cpu = layer_inputs(w)
    ctx = make_ctx(w)
    V = [np.array([5, 300], np.int64)] * 2  # no slash offsets: rows < 5 see nothing
    S = [np.array([], np.int64)] * 2
    out, lse = ctx.sparse_prefill(dev["q"], 0, 640, dev["k"], dev["v"], lists_to_sets(V, S, 640, 640))
    out, lse = f64(out), f64(lse)
    assert np.all(out[:, :5] == 0) and np.all(np.isneginf(lse[:, :5]))
    for h in range(2):
        oo, _ = vo.attention_rows(cpu["q"][h, 5:], np.arange(5, 640), cpu["k"][0], cpu["v"][0], 640,
                                  vo.membership(640, V[h]), vo.membership(640, S[h]), w.rope_base, scale_of(w),
                                  round_out=False)
        assert_outputs_close(out[h, 5:], oo)


def test_sparse_prefill_is_deterministic(case):
    name, w, dca, dev, cpu, ctx = case
    cs, e = _chunks(w)[-1]
    V, S = _random_sets(np.random.default_rng(5), w.hq, e, 0.2, 0.05)
    sets = lists_to_sets(V, S, e, e)
    qc = dev["q"][:, cs:e].contiguous()
    a = [t.clone() for t in ctx.sparse_prefill(qc, cs, e, dev["k"], dev["v"], sets)]
    b = ctx.sparse_prefill(qc, cs, e, dev["k"], dev["v"], sets)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_long_lists_swept_from_a_shared_start():
    """Work lists of 1024 entries or more start where the CTAs of their KV head are
    loading and wrap around. 40 query heads over 8 KV heads, 1024 query rows (4 tile
    pairs) against 132096 keys (1032 blocks): 160 attention CTAs, so those that start
    after the first wave join their KV head's sweep part-way along the list. Three
    launches, each against the oracle on the first and last row of every query tile and
    32 random rows per head; then, with the deterministic switch, two launches bit for
    bit equal."""
    w = small_workload(3, seq_len=132096, chunk=1024, hq=40, hkv=8, n_planted=8)
    st = structure(w)
    cs, e = w.seq_len - w.chunk, w.seq_len
    q = torch.stack([generate_head(w, "q", h, rows=torch.arange(cs, e), st=st) for h in range(w.hq)])
    k = torch.stack([generate_head(w, "k", h, st=st) for h in range(w.hkv)])
    v = torch.stack([generate_head(w, "v", h, st=st) for h in range(w.hkv)])
    dq, dk, dv = q.cuda(), k.cuda(), v.cuda()
    ctx = make_ctx(w)
    V, S = _random_sets(np.random.default_rng(9), w.hq, e, 0.2, 0.05)
    sets = lists_to_sets(V, S, e, e)
    runs = []
    for _ in range(3):
        out, lse = ctx.sparse_prefill(dq, cs, e, dk, dv, sets)
        assert ctx.status() == vsb.VS_OK
        runs.append((f64(out), f64(lse)))
    rng = np.random.default_rng(10)
    starts = np.arange(cs, e, 128)
    rows = np.union1d(np.concatenate([starts, starts + 127]), rng.choice(np.arange(cs, e), 32, replace=False))
    qh, kh, vh = f64(q), f64(k), f64(v)
    for hk in range(w.hkv):
        kr = vo.rope(kh[hk], np.arange(e), w.rope_base)
        for h in range(hk * w.group, (hk + 1) * w.group):
            oo, ol = vo.attention_rows(qh[h, rows - cs], rows, kh[hk], vh[hk], e, vo.membership(e, V[h]),
                                       vo.membership(e, S[h]), w.rope_base, scale_of(w), k_rot=kr,
                                       round_out=False)
            for i, (out, lse) in enumerate(runs):
                assert_outputs_close(out[h, rows - cs], oo, f"run {i} h={h}", w=w)
                assert np.allclose(lse[h, rows - cs], ol, rtol=0, atol=2e-3), (i, h)
    ctx.set_deterministic(True)
    a = [t.clone() for t in ctx.sparse_prefill(dq, cs, e, dk, dv, sets)]
    b = ctx.sparse_prefill(dq, cs, e, dk, dv, sets)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def _check_layer(name, w, keep, ref, out):
    """Per chunk and head: identical sets give outputs within tolerance; sets that
    differ under the same budgets differ only by near-ties; other budgets are only
    allowed where the oracle's refinement met a recall within TAU_SLACK of tau."""
    out = f64(out)
    for kc, rc in zip(keep, ref):
        V, S = sets_to_lists(kc["sets"])
        kv_g, ks_g = kc["kv"].cpu().numpy(), kc["ks"].cpu().numpy()
        for h in range(w.hq):
            r = rc["heads"][h]
            same = np.array_equal(V[h], r["V"]) and np.array_equal(S[h], r["S"])
            if same:
                assert_outputs_close(out[h, rc["cs"] : rc["e"]], r["out"], f"{name} chunk {rc['cs']} h={h}", w=w)
            elif (int(kv_g[h]), int(ks_g[h])) == (int(r["kv"]), int(r["ks"])):
                # same budgets: the sets may differ only by near-ties of the k-th score
                assert_near_tie_equal(V[h], r["V"], r["vert"], int(r["kv"]))
                sl = r["slash"].copy()
                sl[0] = np.inf
                assert_near_tie_equal(S[h], r["S"], sl, int(r["ks"]))
            else:  # other budgets: only a refinement decision at tau may tell them apart
                assert w.refine_tau is not None and any(
                    abs(x - w.refine_tau) < TAU_SLACK for _, _, x in r["trace"]), (name, rc["cs"], h, r["trace"])


def test_layer_prefill_end_to_end(case):
    """The chunk loop on the GPU against the oracle's chunk loop."""
    name, w, dca, dev, cpu, ctx = case
    keep = []
    out = vsb.layer_prefill(ctx, dev["q"], dev["k"], dev["v"], chunk=w.chunk, kv_budget=w.kv_budget,
                            ks_budget=w.ks_budget, tau=w.refine_tau, keep=keep)
    assert ctx.status() == vsb.VS_OK
    ref = vo.layer_prefill(cpu["q"], cpu["k"], cpu["v"], chunk=w.chunk, last_q=w.last_q, kv_budget=w.kv_budget,
                           ks_budget=w.ks_budget, tau=w.refine_tau, base=w.rope_base, scale=scale_of(w), dca=dca,
                           round_out=False)
    _check_layer(name, w, keep, ref, out)


def test_calibrated_budgets_and_fixed_budget_prefill(case):
    """Offline refinement: per-head budgets calibrated on the sequence match the
    oracle's (up to recalls within TAU_SLACK of tau), and the prefill with those
    fixed budgets (selection only, no refinement) matches the oracle's."""
    name, w, dca, dev, cpu, ctx = case
    if w.refine_tau is None:
        pytest.skip("no refinement threshold")
    kv, ks = vsb.calibrate(ctx, dev["q"], dev["k"], chunk=w.chunk, kv_budget=w.kv_budget,
                           ks_budget=w.ks_budget, tau=w.refine_tau)
    assert ctx.status() == vsb.VS_OK
    kw = dict(chunk=w.chunk, last_q=w.last_q, kv_budget=w.kv_budget, ks_budget=w.ks_budget, tau=w.refine_tau,
              base=w.rope_base, scale=scale_of(w))
    okv, oks = vo.calibrate(cpu["q"], cpu["k"], **kw)
    kv_h, ks_h = kv.cpu().numpy(), ks.cpu().numpy()
    if (list(kv_h), list(ks_h)) != (okv, oks):
        traces = vo.layer_prefill(cpu["q"], cpu["k"], cpu["v"], **kw, dca=dca, rows_per_chunk=lambda cs, e: [e - 1])
        for h in range(w.hq):
            if (kv_h[h], ks_h[h]) != (okv[h], oks[h]):
                assert any(abs(x - w.refine_tau) < TAU_SLACK for c in traces for _, _, x in c["heads"][h]["trace"])
    keep = []
    out = vsb.layer_prefill(ctx, dev["q"], dev["k"], dev["v"], chunk=w.chunk, kv_budget=kv, ks_budget=ks,
                            tau=None, keep=keep)
    assert ctx.status() == vsb.VS_OK
    ref = vo.layer_prefill(cpu["q"], cpu["k"], cpu["v"], **{**kw, "kv_budget": kv_h, "ks_budget": ks_h, "tau": None},
                           dca=dca, round_out=False)
    _check_layer(name, w, keep, ref, out)


def test_wait_timeout_is_reported_and_context_survives():
    w = small_workload(2, seq_len=512, chunk=512, hq=2, hkv=1)
    ctx = make_ctx(w)
    assert ctx.status() == vsb.VS_OK
    ctx.selftest_wait_timeout(2_000_000)  # 2 ms
    assert ctx.status() == vsb.VS_ERR_TIMEOUT
    assert ctx.status() == vsb.VS_OK  # cleared
    dev, _ = layer_inputs(w)
    ctx.estimate(dev["q"], 0, dev["k"], 512)
    assert ctx.status() == vsb.VS_OK


def test_host_validation_on_device():
    w = small_workload(2, seq_len=512, chunk=512, hq=2, hkv=1)
    ctx = make_ctx(w)
    dev, _ = layer_inputs(w)
    with pytest.raises(vsb.VsError) as ei:
        ctx.estimate(dev["q"], 0, dev["k"], 513)  # e beyond max_seq
    assert ei.value.status in (vsb.VS_ERR_UNSUPPORTED, vsb.VS_ERR_INVALID_ARG)
    V, S = [np.arange(4)] * 2, [np.arange(1)] * 2
    with pytest.raises(vsb.VsError) as ei:
        ctx.sparse_prefill(dev["q"], 64, 512, dev["k"], dev["v"], lists_to_sets(V, S, 8, 8))  # q_pos0 % 128
    assert ei.value.status == vsb.VS_ERR_UNSUPPORTED
    # a list entry beyond e is caught on the device and reported
    bad = lists_to_sets([np.array([0, 600])] * 2, S, 8, 8)
    ctx.sparse_prefill(dev["q"], 0, 512, dev["k"], dev["v"], bad)
    assert ctx.status() == vsb.VS_ERR_DEVICE_CHECK


def test_dca_with_chunk_beyond_sequence_equals_continuous_rope():
    """DCA whose chunk covers the sequence reduces to plain RoPE: the GPU path
    with DCA gives the same outputs as without it (bit-identical)."""
    w = small_workload(2, seq_len=900, chunk=512, hq=4, hkv=2)
    dev, _ = layer_inputs(w)
    V, S = _random_sets(np.random.default_rng(9), w.hq, w.seq_len, 0.2, 0.05)
    outs = []
    for dca in (None, (1152, 128)):  # S = 1024 >= 900
        ctx = make_ctx(w, max_chunk=w.chunk, dca=dca)
        out = torch.zeros_like(dev["q"])
        for cs, e in _chunks(w):
            sets = lists_to_sets([x[x < e] for x in V], [x[x < e] for x in S], e, e)
            ctx.sparse_prefill(dev["q"], cs, e, dev["k"], dev["v"], sets, out=out, full=True)
        assert ctx.status() == vsb.VS_OK
        outs.append(out)
    assert torch.equal(outs[0], outs[1])


def test_empty_and_out_of_range_sizes_are_rejected():
    w = small_workload(2, seq_len=512, chunk=512, hq=2, hkv=1)
    dev, _ = layer_inputs(w)
    ctx = make_ctx(w, max_chunk=256)
    with pytest.raises(vsb.VsError):
        ctx.estimate(dev["q"], 0, dev["k"], 0)
    buf = torch.empty(2, 64, dtype=torch.float32, device="cuda")
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    for e in (0, -1, 513):  # empty, negative, beyond max_seq
        st = ctx.lib.vs_estimate(ctx.handle, p(dev["q"]), 512, 0, p(dev["k"]), 512, e, p(buf), p(buf), 64, p(buf),
                                 None)
        assert st in (vsb.VS_ERR_INVALID_ARG, vsb.VS_ERR_UNSUPPORTED), (e, st)
    with pytest.raises(vsb.VsError):  # a chunk of 512 rows, longer than max_chunk = 256
        ctx.sparse_prefill(dev["q"], 0, 512, dev["k"], dev["v"], lists_to_sets([np.arange(4)] * 2, [np.arange(1)] * 2, 8, 8))
    assert ctx.status() == vsb.VS_OK


@pytest.mark.parametrize("heads", [(4, 2), (40, 8)])
@pytest.mark.parametrize("dca", [None, (2048, 256)])
def test_sparse_prefill_gathers_scattered_verticals(dca, heads):
    """A band of slash offsets plus scattered vertical columns (before each chunk and
    inside it), the shape in which the kernel gathers vertical columns into dense
    groups instead of executing their key blocks: every row against the oracle (with
    40 heads, the first and last row of every query tile and 64 random rows per chunk),
    and the executed tiles far below the causal dense count. With DCA (stride 1792) the
    groups are split at DCA chunk boundaries, each with its own query rotation. 40 heads
    give 320 attention CTAs per chunk, more than two waves of one CTA per SM, so lists
    swept from their end (every other wave) are covered too."""
    hq, hkv = heads
    w = small_workload(2, seq_len=6144, chunk=2048, hq=hq, hkv=hkv, n_planted=8)
    dev, cpu = layer_inputs(w)
    ctx = make_ctx(w, dca=dca)
    rng = np.random.default_rng(21)
    e_all = w.seq_len
    V = []
    for h in range(w.hq):
        cols = rng.choice(e_all, 220, replace=False)
        cols = np.union1d(cols, np.arange(640, 768))  # one full key block: executed, never gathered
        V.append(cols.astype(np.int64))
    S = [np.union1d(np.arange(0, 300), rng.choice(np.arange(300, e_all), 3, replace=False)).astype(np.int64)
         for _ in range(w.hq)]
    scale = scale_of(w)
    dense_tiles = 0
    executed = 0
    for cs, e in _chunks(w):
        sets = lists_to_sets([x[x < e] for x in V], [x[x < e] for x in S], e, e)
        out = torch.zeros_like(dev["q"])
        ctx.sparse_prefill(dev["q"], cs, e, dev["k"], dev["v"], sets, out=out, full=True)
        assert ctx.status() == vsb.VS_OK
        ex, _ = ctx.prefill_stats()
        executed += ex
        dense_tiles += w.hq * sum((r0 // 128 + 1) for r0 in range(cs, e, 128))
        rows = np.arange(cs, e)
        if w.hq > 4:
            tile_ends = np.concatenate([np.arange(cs, e, 128), np.minimum(np.arange(cs, e, 128) + 127, e - 1)])
            rows = np.union1d(tile_ends, rng.choice(rows, 64, replace=False))
        got = f64(out[:, rows])
        for h in range(w.hq):
            vh, sh = V[h][V[h] < e], S[h][S[h] < e]
            oo, _ = vo.attention_rows(cpu["q"][h, rows], rows, cpu["k"][h // w.group], cpu["v"][h // w.group], e,
                                      vo.membership(e, vh), vo.membership(e, sh), w.rope_base, scale, dca,
                                      round_out=False)
            assert_outputs_close(got[h], oo, f"gather dca={dca} hq={w.hq} cs={cs} h={h}", w=w)
    assert executed < 0.5 * dense_tiles, (executed, dense_tiles)


def test_rewritten_keys_under_a_cached_rotation_are_reported():
    """The context caches rotated keys per K pointer; keys rewritten in place without
    vs_context_reset are caught by the sampled re-rotation of a reused cache."""
    w = small_workload(2, seq_len=1024, chunk=1024, hq=2, hkv=1)
    dev, _ = layer_inputs(w)
    for dca in (None, (512, 128)):
        ctx = make_ctx(w, dca=dca)
        V, S = [np.arange(0, 1024, 3)] * 2, [np.arange(8)] * 2
        sets = lists_to_sets(V, S, 1024, 1024)
        k = dev["k"].clone()
        ctx.estimate(dev["q"], 0, k, 1024)
        ctx.sparse_prefill(dev["q"], 0, 1024, k, dev["v"], sets)
        assert ctx.status() == vsb.VS_OK
        ctx.estimate(dev["q"], 0, k, 1024)  # reuses both caches: unchanged keys pass
        ctx.sparse_prefill(dev["q"], 0, 1024, k, dev["v"], sets)
        assert ctx.status() == vsb.VS_OK
        k.mul_(2.0)  # another sequence in the same buffer, without a reset
        ctx.estimate(dev["q"], 0, k, 1024)
        assert ctx.status() == vsb.VS_ERR_DEVICE_CHECK
        assert b"keys changed" in ctx.lib.vs_last_error()
        ctx.reset()
        ctx.estimate(dev["q"], 0, k, 1024)
        ctx.sparse_prefill(dev["q"], 0, 1024, k, dev["v"], sets)
        assert ctx.status() == vsb.VS_OK
