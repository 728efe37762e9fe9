"""Pins of the CPU oracle against things other than itself (CPU only).

Each test ties an oracle function to brute force (tests/bruteforce.py, written
separately in pure Python), a closed form, an invariant, a special case that
reduces to a library routine, or the hand-worked DCA table in tests/golden/.
`test_planted_mistakes` checks that plausible slips in the oracle are caught.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import vs_oracle as vo
from tests import bruteforce as bf

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
BASE = 1.0e7


def _bf16_array(rng, shape, scale=1.0):
    x = torch.tensor(rng.standard_normal(shape) * scale, dtype=torch.float32).to(torch.bfloat16)
    return x.to(torch.float64).numpy()


# ------------------------------------------------------------------ bf16 rounding
def test_bf16_rne_matches_frexp_bruteforce(rng):
    x = rng.standard_normal(4000) * np.exp(rng.uniform(-20, 20, 4000))
    got = vo.bf16_rne(x)
    want = np.array([bf.bf16(float(t)) for t in x])
    assert np.array_equal(got, want)


def test_bf16_rne_matches_torch_on_float32_values(rng):
    # torch rounds float32 -> bfloat16 to nearest even; on float32-exact inputs
    # the float64 rounding must agree
    x32 = (rng.standard_normal(20000) * 7).astype(np.float32)
    want = torch.from_numpy(x32).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(vo.bf16_rne(x32.astype(np.float64)), want)


def test_bf16_rne_ties_go_to_even():
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: the even neighbour is 1
    assert vo.bf16_rne(np.array([1.0 + 2.0 ** -8]))[0] == 1.0
    # 1 + 3 * 2^-8 is halfway between 1 + 2^-7 and 1 + 2^-6: even is 1 + 2^-6
    assert vo.bf16_rne(np.array([1.0 + 3 * 2.0 ** -8]))[0] == 1.0 + 2.0 ** -6


# ------------------------------------------------------------------ RoPE
@pytest.mark.parametrize("d", [8, 16, 128])
def test_rope_matches_bruteforce(rng, d):
    x = _bf16_array(rng, (6, d))
    pos = np.array([0, 1, 5, 1000, 65535, 1048575])
    got = vo.rope(x, pos, BASE)
    for r in range(6):
        want = bf.rope_row(list(x[r]), int(pos[r]), BASE)
        assert np.array_equal(got[r], np.array(want))


def test_rope_inverse_frequencies_closed_form():
    th = vo.inv_freq(128, BASE)
    assert th[0] == 1.0
    assert th[32] == pytest.approx(BASE ** -0.5, rel=1e-15)
    assert th[63] == pytest.approx(BASE ** (-126 / 128), rel=1e-15)
    assert np.all(np.diff(th) < 0)


def test_rope_position_zero_is_identity(rng):
    x = _bf16_array(rng, (5, 128))
    assert np.array_equal(vo.rope(x, np.zeros(5, dtype=int), BASE), x)


def test_rope_preserves_pair_norms(rng):
    x = _bf16_array(rng, (4, 16))
    y = vo.rope(x, np.array([3, 77, 4096, 999999]), BASE, round_bf16=False)
    n0 = x[:, :8] ** 2 + x[:, 8:] ** 2
    n1 = y[:, :8] ** 2 + y[:, 8:] ** 2
    assert np.allclose(n0, n1, rtol=1e-13, atol=0)


def test_rope_scores_depend_only_on_relative_position(rng):
    # RoPE relativity: q(i+t).k(j+t) == q(i).k(j) (unrounded, float64)
    q = _bf16_array(rng, (1, 128))
    k = _bf16_array(rng, (1, 128))
    for i, j, t in [(10, 3, 1000), (500000, 499000, 123456), (7, 7, 999999)]:
        s0 = vo.rope(q, [i], BASE, False) @ vo.rope(k, [j], BASE, False).T
        s1 = vo.rope(q, [i + t], BASE, False) @ vo.rope(k, [j + t], BASE, False).T
        assert abs(s0 - s1).item() <= 1e-9 * max(1.0, abs(s0).item())


# ------------------------------------------------------------------ estimation
@pytest.mark.parametrize("nr,e,d", [(5, 20, 8), (3, 3, 16), (8, 33, 16)])
def test_estimate_matches_bruteforce(rng, nr, e, d):
    q = _bf16_array(rng, (nr, d))
    k = _bf16_array(rng, (e, d))
    scale = 1 / math.sqrt(d)
    lse, vert, slash, a = vo.estimate(q, k, e, BASE, scale)
    blse, bvert, bslash, bA = bf.estimate([list(r) for r in q], [list(r) for r in k], e, BASE, scale)
    assert np.allclose(lse, blse, rtol=1e-12, atol=1e-12)
    assert np.allclose(vert, bvert, rtol=1e-12, atol=1e-15)
    assert np.allclose(slash, bslash, rtol=1e-12, atol=1e-15)
    assert np.allclose(a, np.array(bA), rtol=1e-12, atol=1e-15)


def test_estimate_with_prerotated_keys_is_identical(rng):
    q = _bf16_array(rng, (7, 128), 1.5)
    k = _bf16_array(rng, (300, 128), 1.5)
    kr = vo.rope(k, np.arange(300), BASE)
    for e in (7, 123, 300):
        a = vo.estimate(q, k, e, BASE, 0.1)
        b = vo.estimate(q, None, e, BASE, 0.1, k_rot=kr)
        for x, y in zip(a, b):
            assert np.array_equal(x, y)


def test_row_softmax_sums_to_one(rng):
    q = _bf16_array(rng, (64, 128))
    k = _bf16_array(rng, (700, 128))
    _, _, _, a = vo.estimate(q, k, 700, BASE, 1 / math.sqrt(128))
    assert np.all(np.abs(a.sum(axis=1) - 1.0) <= 1e-12)


def test_vertical_and_slash_mass_equal_row_count(rng):
    q = _bf16_array(rng, (64, 128))
    k = _bf16_array(rng, (500, 128))
    _, vert, slash, _ = vo.estimate(q, k, 500, BASE, 1 / math.sqrt(128))
    assert abs(vert.sum() - 64) <= 1e-12 * 64
    assert abs(slash.sum() - 64) <= 1e-12 * 64
    # causal: no estimation row reaches beyond itself, so offsets >= 0 only
    assert np.all(vert >= 0) and np.all(slash >= 0)


def test_estimate_uniform_scores_closed_form():
    # q = 0 gives equal scores: row i spreads 1/(i+1) over keys 0..i
    nr, e, d = 4, 10, 8
    q = np.zeros((nr, d))
    k = np.ones((e, d))
    lse, vert, slash, _ = vo.estimate(q, k, e, BASE, 0.3)
    rows = range(e - nr, e)
    assert np.allclose(lse, [math.log(i + 1) for i in rows], rtol=0, atol=1e-14)
    want_v = [sum(1 / (i + 1) for i in rows if j <= i) for j in range(e)]
    assert np.allclose(vert, want_v, atol=1e-14)
    want_s = [sum(1 / (i + 1) for i in rows if i - dd >= 0) for dd in range(e)]
    assert np.allclose(slash, want_s, atol=1e-14)


# ------------------------------------------------------------------ selection
def test_topk_matches_sorted_with_ties(rng):
    s = rng.integers(0, 5, 200).astype(np.float64)  # many ties
    for k in [1, 7, 50, 200, 500]:
        want = sorted(sorted(range(200), key=lambda j: (-s[j], j))[: min(k, 200)])
        assert list(vo.topk_sorted(s, k)) == want


def test_topk_matches_numpy_stable_argsort(rng):
    s = rng.standard_normal(1000)
    s[::7] = 0.25  # ties
    order = np.argsort(-s, kind="stable")  # stable: equal scores keep index order
    for k in [10, 333]:
        assert np.array_equal(vo.topk_sorted(s, k), np.sort(order[:k]))


def test_kth_score_matches_stable_sort_with_ties(rng):
    """kth_score is the score at rank k of the (score descending, index ascending)
    order: checked against Python's stable sort on integer scores with many ties,
    k capped at the length, and the set property around it (fewer than k scores
    above the k-th, at least k at or above it)."""
    s = rng.integers(0, 6, 300).astype(np.float64) / 4.0
    order = sorted(range(300), key=lambda j: (-s[j], j))
    for k in [1, 2, 17, 150, 299, 300, 1000]:
        kk = min(k, 300)
        want = s[order[kk - 1]]
        got = vo.kth_score(s, k)
        assert got == want, (k, got, want)
        assert np.sum(s > got) < kk <= np.sum(s >= got)
        assert vo.kth_score(s, k, order=vo.ranking(s)) == want
    # a strictly increasing score: the k-th largest is the (n - k)-th element
    inc = np.arange(50, dtype=np.float64)
    assert vo.kth_score(inc, 5) == 45.0


def test_select_with_precomputed_orders_is_identical(rng):
    vert = rng.integers(0, 9, 500).astype(np.float64)
    slash = rng.integers(0, 9, 500).astype(np.float64)
    orders = vo.select_orders(vert, slash)
    for kv, ks in [(1, 1), (37, 81), (500, 500), (900, 3)]:
        a = vo.select(vert, slash, kv, ks)
        b = vo.select(vert, slash, kv, ks, orders)
        assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_select_matches_bruteforce_and_forces_offset0(rng):
    vert = rng.random(64)
    slash = rng.random(64)
    slash[0] = 0.0  # the smallest score, still selected
    V, S = vo.select(vert, slash, 9, 5)
    bV, bS = bf.select(list(vert), list(slash), 9, 5)
    assert list(V) == bV and list(S) == bS
    assert 0 in S and len(S) == 5 and np.all(np.diff(S) > 0)


# ------------------------------------------------------------------ recall and refinement
def _tiny_estimation(rng, nr=6, e=40, d=16):
    q = _bf16_array(rng, (nr, d), 2.0)
    k = _bf16_array(rng, (e, d), 2.0)
    return vo.estimate(q, k, e, BASE, 1 / math.sqrt(d))


def test_recall_is_exp_of_lse_difference(rng):
    # Attention_Recall = exp(lse_sparse - lse_full), computed here from the raw
    # scores restricted to the selected keys
    nr, e, d = 6, 40, 16
    q = _bf16_array(rng, (nr, d), 2.0)
    k = _bf16_array(rng, (e, d), 2.0)
    scale = 1 / math.sqrt(d)
    lse, vert, slash, a = vo.estimate(q, k, e, BASE, scale)
    V, S = vo.select(vert, slash, 7, 4)
    inV, inS = vo.membership(e, V), vo.membership(e, S)
    rows = np.arange(e - nr, e)
    kr = vo.rope(k, np.arange(e), BASE)
    per = []
    for r, i in enumerate(rows):
        qi = vo.rope(q[r : r + 1], [i], BASE)[0]
        js = [j for j in range(i + 1) if inV[j] or inS[i - j]]
        s = scale * (kr[js] @ qi)
        lse_sparse = s.max() + math.log(np.exp(s - s.max()).sum())
        per.append(math.exp(lse_sparse - lse[r]))
    assert vo.recall(a, rows, inV, inS) == pytest.approx(np.mean(per), rel=1e-12)


@pytest.mark.parametrize("kv,ks", [(3, 2), (7, 4), (20, 30), (40, 40)])
def test_recall_is_vertical_plus_slash_mass_minus_their_overlap(rng, kv, ks):
    # The mass of the selected elements is the mass of the selected columns (their
    # vertical sums) plus that of the selected offsets (their slash sums), minus the
    # elements both select, counted twice: the identity by which the recall at the
    # base budgets is taken from the estimation pass's sums.
    lse, vert, slash, a = _tiny_estimation(rng)
    e, nr = vert.shape[0], a.shape[0]
    rows = np.arange(e - nr, e)
    V, S = vo.select(vert, slash, kv, ks)
    inV, inS = vo.membership(e, V), vo.membership(e, S)
    both = 0.0
    for r, i in enumerate(rows):
        for j in range(int(i) + 1):
            if inV[j] and inS[int(i) - j]:
                both += a[r, j]
    mass = vert[inV].sum() + slash[inS].sum() - both
    assert vo.recall(a, rows, inV, inS) == pytest.approx(mass / nr, rel=1e-12, abs=1e-15)


def test_recall_full_mask_is_one_and_monotone(rng):
    lse, vert, slash, a = _tiny_estimation(rng)
    e = vert.shape[0]
    rows = np.arange(e - a.shape[0], e)
    full = np.ones(e, dtype=bool)
    assert vo.recall(a, rows, full, full) == pytest.approx(1.0, abs=1e-12)
    prev = -1.0
    kv, ks = 2, 1
    while True:
        V, S = vo.select(vert, slash, kv, ks)
        rc = vo.recall(a, rows, vo.membership(e, V), vo.membership(e, S))
        assert rc >= prev - 1e-15
        prev = rc
        if kv >= e and ks >= e:
            break
        kv, ks = min(2 * kv, e), min(2 * ks, e)
    assert prev == pytest.approx(1.0, abs=1e-12)


@pytest.mark.parametrize("tau", [0.3, 0.6, 0.95, 1.5])
def test_refine_matches_bruteforce(rng, tau):
    nr, e, d = 6, 40, 16
    q = _bf16_array(rng, (nr, d), 2.0)
    k = _bf16_array(rng, (e, d), 2.0)
    scale = 1 / math.sqrt(d)
    _, vert, slash, a = vo.estimate(q, k, e, BASE, scale)
    rows = np.arange(e - nr, e)
    kv, ks, V, S, rc, trace = vo.refine(a, rows, vert, slash, 2, 1, tau)
    bkv, bks, bV, bS, brc = bf.refine([list(r) for r in a], list(rows), list(vert), list(slash), 2, 1, tau)
    assert (kv, ks) == (bkv, bks) and list(V) == bV and list(S) == bS
    assert rc == pytest.approx(brc, rel=1e-12)
    if tau > 1:
        assert kv == e and ks == e  # saturates


# ------------------------------------------------------------------ attention
def _sdpa_causal(q, k, v, scale):
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x))[None, None]
    o = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), is_causal=True, scale=scale)
    return o[0, 0].numpy()


def test_full_mask_equals_dense_causal_attention(rng):
    n, d = 150, 16
    q = _bf16_array(rng, (n, d))
    k = _bf16_array(rng, (n, d))
    v = _bf16_array(rng, (n, d))
    scale = 1 / math.sqrt(d)
    full = np.ones(n, dtype=bool)
    rows = np.arange(n)
    o, _ = vo.attention_rows(q, rows, k, v, n, full, full, BASE, scale)
    od, _ = vo.attention_rows_dense(q, rows, k, v, n, full, full, BASE, scale)
    qr, kr = vo.rope(q, rows, BASE), vo.rope(k, rows, BASE)
    want = vo.bf16_rne(_sdpa_causal(qr, kr, v, scale))
    ulp = 2.0 ** -7 * np.maximum(np.abs(want), 2.0 ** -20)
    assert np.all(np.abs(o - want) <= ulp) and np.mean(o == want) > 0.99
    assert np.array_equal(o, od)


@pytest.mark.parametrize("dca", [None, (16, 4), (24, 6)])
def test_attention_matches_bruteforce(rng, dca):
    n, d = 40, 8
    q = _bf16_array(rng, (n, d), 1.5)
    k = _bf16_array(rng, (n, d), 1.5)
    v = _bf16_array(rng, (n, d))
    scale = 1 / math.sqrt(d)
    V = np.array([1, 5, 6, 20, 33])
    S = np.array([0, 2, 9, 17])
    rows = np.arange(20, 40)
    o, lse = vo.attention_rows(q[rows], rows, k, v, n, vo.membership(n, V), vo.membership(n, S),
                               BASE, scale, dca)
    bo, blse = bf.attention([list(r) for r in q[rows]], list(rows), [list(r) for r in k],
                            [list(r) for r in v], n, list(V), list(S), BASE, scale, dca)
    assert np.allclose(lse, blse, rtol=1e-12, atol=1e-12)
    bo = np.array(bo)
    assert np.all(np.abs(o - bo) <= 2.0 ** -7 * np.abs(bo) + 1e-30)
    assert np.mean(o == bo) > 0.95


@pytest.mark.parametrize("dca", [None, (64, 8)])
def test_block_evaluator_equals_row_definition(rng, dca):
    n, d = 300, 16
    q = _bf16_array(rng, (n, d))
    k = _bf16_array(rng, (n, d))
    v = _bf16_array(rng, (n, d))
    inV = rng.random(n) < 0.2
    inS = rng.random(n) < 0.1
    inS[0] = True
    rows = np.arange(37, 300)
    o1, l1 = vo.attention_rows(q[rows], rows, k, v, n, inV, inS, BASE, 0.25, dca, block=64)
    o2, l2 = vo.attention_rows_dense(q[rows], rows, k, v, n, inV, inS, BASE, 0.25, dca)
    assert np.allclose(l1, l2, rtol=1e-13, atol=1e-13)
    assert np.array_equal(o1, o2) or np.max(np.abs(o1 - o2)) <= 2.0 ** -7 * np.max(np.abs(o2))


@pytest.mark.parametrize("dca", [None, (64, 8)])
def test_attention_rows_unrounded_and_prerotated_paths(rng, dca):
    """round_out=False returns the float64 outputs whose bf16 rounding is the
    default output; pre-rotated keys at the key positions change nothing."""
    e = 150
    q = _bf16_array(rng, (e, 16))
    k = _bf16_array(rng, (e, 16))
    v = _bf16_array(rng, (e, 16))
    inV = rng.random(e) < 0.3
    inS = rng.random(e) < 0.2
    inS[0] = True
    rows = np.array([0, 3, 64, 100, 149])
    o, l = vo.attention_rows(q[rows], rows, k, v, e, inV, inS, BASE, 0.25, dca)
    ox, lx = vo.attention_rows(q[rows], rows, k, v, e, inV, inS, BASE, 0.25, dca, round_out=False)
    assert np.array_equal(vo.bf16_rne(ox), o) and np.array_equal(l, lx)
    assert not np.array_equal(ox, o)  # the unrounded values carry more bits
    kr = vo.rope(k, vo.key_positions(e, dca), BASE)
    o2, l2 = vo.attention_rows(q[rows], rows, None, v, e, inV, inS, BASE, 0.25, dca, k_rot=kr)
    assert np.array_equal(o2, o) and np.array_equal(l2, l)


def test_uniform_scores_average_selected_values(rng):
    # q = 0: every selected key gets the same weight, O_i = mean of selected v_j
    n, d = 50, 8
    q = np.zeros((n, d))
    k = _bf16_array(rng, (n, d))
    v = _bf16_array(rng, (n, d))
    inV = np.zeros(n, dtype=bool)
    inV[[3, 10]] = True
    inS = np.zeros(n, dtype=bool)
    inS[[0, 4]] = True
    rows = np.array([12, 40])
    o, lse = vo.attention_rows(q[rows], rows, k, v, n, inV, inS, BASE, 0.3)
    for r, i in enumerate(rows):
        js = sorted({3, 10, i, i - 4} & set(range(i + 1)))
        assert lse[r] == pytest.approx(math.log(len(js)), abs=1e-14)
        assert np.allclose(o[r], vo.bf16_rne(v[js].mean(axis=0)), atol=0)


# ------------------------------------------------------------------ DCA
def test_dca_golden_table():
    with open(os.path.join(GOLDEN, "dca_positions_C8_W2.json")) as f:
        g = json.load(f)
    C, W = g["C"], g["W"]
    for c in g["cases"]:
        pq, pk = vo.dca_positions(c["i"], [c["j"]], C, W)
        assert (int(pq[0]), int(pk[0])) == (c["pq"], c["pk"]), c
        assert int(pq[0] - pk[0]) == c["rel"]


def test_dca_statements_on_random_pairs(rng):
    for C, W in [(64, 8), (65536, 2048), (262144, 8192)]:
        S = C - W
        i = rng.integers(0, 5 * C, 4000)
        j = (i - rng.integers(0, 5 * C, 4000)).clip(0)
        for a, b in zip(i, j):
            pq, pk = vo.dca_positions(int(a), [int(b)], C, W)
            rel = int(pq[0] - pk[0])
            assert 0 <= rel <= C - 1  # never beyond the pretraining length
            if a // S == b // S:
                assert rel == a - b  # intra keeps the true distance
            elif a // S == b // S + 1 and a % S < W:
                assert rel == a - b  # successive, inside the local window


def test_dca_reduces_to_rope_when_chunk_covers_sequence(rng):
    n, d = 200, 16
    q = _bf16_array(rng, (n, d))
    k = _bf16_array(rng, (n, d))
    v = _bf16_array(rng, (n, d))
    inV = rng.random(n) < 0.3
    inS = rng.random(n) < 0.2
    inS[0] = True
    rows = np.arange(n)
    o0, l0 = vo.attention_rows(q, rows, k, v, n, inV, inS, BASE, 0.25, None)
    o1, l1 = vo.attention_rows(q, rows, k, v, n, inV, inS, BASE, 0.25, (n + 32, (n + 32) // 32))
    assert np.array_equal(o0, o1) and np.array_equal(l0, l1)


# ------------------------------------------------------------------ chunking and GQA
def _layer(rng, hq, hkv, n, d):
    return (_bf16_array(rng, (hq, n, d)), _bf16_array(rng, (hkv, n, d)), _bf16_array(rng, (hkv, n, d)))


def test_chunked_equals_unchunked_under_full_mask(rng):
    q, k, v = _layer(rng, 2, 1, 96, 16)
    kw = dict(last_q=8, kv_budget=10 ** 6, ks_budget=10 ** 6, tau=None, base=BASE)
    a = vo.layer_prefill(q, k, v, chunk=96, **kw)
    b = vo.layer_prefill(q, k, v, chunk=32, **kw)
    for h in range(2):
        ob = np.concatenate([c["heads"][h]["out"] for c in b])
        assert np.array_equal(a[0]["heads"][h]["out"], ob)


def test_gqa_equals_explicitly_repeated_kv(rng):
    q, k, v = _layer(rng, 4, 2, 64, 16)
    kw = dict(chunk=32, last_q=8, kv_budget=6, ks_budget=5, tau=0.8, base=BASE)
    a = vo.layer_prefill(q, k, v, **kw)
    b = vo.layer_prefill(q, np.repeat(k, 2, axis=0), np.repeat(v, 2, axis=0), **kw)
    for ca, cb in zip(a, b):
        for h in range(4):
            for key in ("out", "lse", "vert", "slash", "V", "S"):
                assert np.array_equal(ca["heads"][h][key], cb["heads"][h][key])


def test_layer_prefill_matches_bruteforce_chain(rng):
    # estimation -> refinement -> attention for two chunks, DCA on
    hq, n, d = 1, 48, 8
    q, k, v = _layer(rng, hq, 1, n, d)
    scale = 1 / math.sqrt(d)
    dca = (20, 4)
    res = vo.layer_prefill(q, k, v, chunk=24, last_q=6, kv_budget=3, ks_budget=2, tau=0.7, base=BASE,
                           scale=scale, dca=dca)
    for c in res:
        cs, e = c["cs"], c["e"]
        r = c["heads"][0]
        est_q = [list(x) for x in q[0, e - 6 : e]]
        _, vert, slash, A = bf.estimate(est_q, [list(x) for x in k[0]], e, BASE, scale)
        kv, ks, V, S, rc = bf.refine(A, list(range(e - 6, e)), vert, slash, 3, 2, 0.7)
        assert (r["kv"], r["ks"]) == (kv, ks) and list(r["V"]) == V and list(r["S"]) == S
        rows = list(range(cs, e))
        o, lse = bf.attention([list(x) for x in q[0, cs:e]], rows, [list(x) for x in k[0]],
                              [list(x) for x in v[0]], e, V, S, BASE, scale, dca)
        assert np.allclose(r["lse"], lse, rtol=1e-12, atol=1e-12)
        assert np.all(np.abs(r["out"] - np.array(o)) <= 2.0 ** -7 * np.abs(np.array(o)) + 1e-30)


def test_calibration_budgets(rng):
    """Offline refinement: on one chunk the calibrated budgets are the refined ones
    (brute-force chain); over several chunks each head keeps the largest refined
    budgets, and with them every chunk's recall reaches tau or both budgets cover
    the chunk's keys (recall is non-decreasing in the budgets)."""
    hq, n, d = 2, 72, 8
    q, k, v = _layer(rng, hq, 1, n, d)
    scale = 1 / math.sqrt(d)
    kw = dict(last_q=6, kv_budget=2, ks_budget=1, tau=0.75, base=BASE, scale=scale)
    kv1, ks1 = vo.calibrate(q[:, :24], k[:, :24], chunk=24, **kw)
    for h in range(hq):
        est_q = [list(x) for x in q[h, 18:24]]
        _, vert, slash, A = bf.estimate(est_q, [list(x) for x in k[0, :24]], 24, BASE, scale)
        bkv, bks, _, _, _ = bf.refine(A, list(range(18, 24)), vert, slash, 2, 1, 0.75)
        assert (kv1[h], ks1[h]) == (bkv, bks)
    kv, ks = vo.calibrate(q, k, chunk=24, **kw)
    per_chunk = vo.layer_prefill(q, k, v, chunk=24, **{**kw, "tau": 0.75})
    for h in range(hq):
        assert kv[h] == max(c["heads"][h]["kv"] for c in per_chunk)
        assert ks[h] == max(c["heads"][h]["ks"] for c in per_chunk)
    fixed = vo.layer_prefill(q, k, v, chunk=24, **{**kw, "kv_budget": kv, "ks_budget": ks, "tau": None})
    for c in fixed:
        for h in range(hq):
            r = c["heads"][h]
            assert r["recall"] >= 0.75 - 1e-12 or (r["kv"] >= c["e"] and r["ks"] >= c["e"])
            assert r["kv"] == min(kv[h], c["e"]) and r["ks"] == min(ks[h], c["e"])


def test_estimation_at_dca_positions(rng):
    """Recall-at-DCA-positions variant: the estimation rows' DCA attention has the
    lse of the dense full-mask DCA attention of the same rows (an independent code
    path), rows sum to one, and with C >= N every pair keeps its continuous
    positions, so it equals the continuous estimation exactly."""
    n, d, nr = 90, 16, 6
    q = _bf16_array(rng, (nr, d), 2.0)
    k = _bf16_array(rng, (n, d), 2.0)
    v = _bf16_array(rng, (n, d))
    scale = 1 / math.sqrt(d)
    rows = np.arange(n - nr, n)
    dca = (40, 8)
    lse, a = vo.estimate_probs_dca(q, k, n, BASE, scale, dca)
    assert np.allclose(a.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    full = np.ones(n, dtype=bool)
    _, lse_att = vo.attention_rows_dense(q, rows, k, v, n, full, full, BASE, scale, dca)
    assert np.allclose(lse, lse_att, rtol=0, atol=1e-12)
    lse_c, _, _, a_c = vo.estimate(q, k, n, BASE, scale)
    lse_w, a_w = vo.estimate_probs_dca(q, k, n, BASE, scale, (128, 16))
    assert np.array_equal(a_w, a_c) and np.array_equal(lse_w, lse_c)
    assert not np.allclose(a, a_c, rtol=0, atol=1e-6)  # DCA positions do change the scores


# ------------------------------------------------------------------ sensitivity
MUTANTS = {
    "rope_sign": lambda x1, x2, c, s: (x1 * c + x2 * s, x2 * c - x1 * s),
    "rope_swap": lambda x1, x2, c, s: (x2 * c - x1 * s, x1 * c + x2 * s),
}


def _mutant_rope(kind):
    f = MUTANTS[kind]

    def rope(x, pos, base, round_bf16=True):
        x = np.asarray(x, dtype=np.float64)
        n, d = x.shape
        p = np.asarray(pos, dtype=np.float64).reshape(n, 1)
        ang = p * vo.inv_freq(d, base).reshape(1, d // 2)
        a, b = f(x[:, : d // 2], x[:, d // 2 :], np.cos(ang), np.sin(ang))
        y = np.concatenate([a, b], axis=1)
        return vo.bf16_rne(y) if round_bf16 else y

    return rope


def _mutant_estimate_offbyone(q_rows, k, e, base, scale):
    lse, vert, slash, a = ORIG_ESTIMATE(q_rows, k, e, base, scale)
    slash = np.roll(slash, 1)  # offsets shifted by one
    return lse, vert, slash, a


def _mutant_estimate_nocausal(q_rows, k, e, base, scale):
    nr = q_rows.shape[0]
    qr = vo.rope(q_rows, np.arange(e - nr, e), base)
    kr = vo.rope(k[:e], np.arange(e), base)
    s = scale * (qr @ kr.T)
    lse = s.max(1) + np.log(np.exp(s - s.max(1, keepdims=True)).sum(1))
    a = np.exp(s - lse[:, None])
    slash = np.zeros(e)
    for r, i in enumerate(range(e - nr, e)):
        slash[: i + 1] += a[r, i::-1]
    return lse, a.sum(0), slash, a


ORIG_ESTIMATE = vo.estimate


@pytest.mark.parametrize("mutant", ["rope_sign", "rope_swap", "slash_offbyone", "no_causal",
                                    "topk_ascending", "ranking_ascending", "ranking_index_descending",
                                    "recall_forward_offsets", "dca_no_clip"])
def test_planted_mistakes_are_caught(rng, monkeypatch, mutant):
    if mutant.startswith("rope"):
        monkeypatch.setattr(vo, "rope", _mutant_rope(mutant))
    elif mutant == "slash_offbyone":
        monkeypatch.setattr(vo, "estimate", _mutant_estimate_offbyone)
    elif mutant == "no_causal":
        monkeypatch.setattr(vo, "estimate", _mutant_estimate_nocausal)
    elif mutant == "topk_ascending":
        monkeypatch.setattr(vo, "topk_sorted",
                            lambda s, k, order=None: np.sort(np.lexsort((np.arange(len(s)), s))[: min(k, len(s))]))
    elif mutant == "ranking_ascending":
        monkeypatch.setattr(vo, "ranking", lambda s: np.lexsort((np.arange(len(s)), s)))
    elif mutant == "ranking_index_descending":
        monkeypatch.setattr(vo, "ranking", lambda s: np.lexsort((-np.arange(len(s)), -s)))
    elif mutant == "recall_forward_offsets":
        def recall(a, rows, inV, inS):  # offsets read forwards: inS[j] instead of inS[i - j]
            tot = 0.0
            for r, i in enumerate(rows):
                sel = inV[: i + 1] | inS[: i + 1]
                tot += a[r, : i + 1][sel].sum()
            return tot / len(rows)
        monkeypatch.setattr(vo, "recall", recall)
    elif mutant == "dca_no_clip":
        monkeypatch.setattr(vo, "dca_q_position",
                            lambda i, c, C, W: [i % (C - W), i % (C - W) + C - W, C - 1][c])
    pins = [
        lambda: test_rope_matches_bruteforce(rng, 16),
        lambda: test_estimate_matches_bruteforce(rng, 5, 20, 8),
        lambda: test_vertical_and_slash_mass_equal_row_count(rng),
        lambda: test_topk_matches_sorted_with_ties(rng),
        lambda: test_select_matches_bruteforce_and_forces_offset0(rng),
        lambda: test_attention_matches_bruteforce(rng, (24, 6)),
        lambda: test_dca_golden_table(),
        lambda: test_dca_statements_on_random_pairs(rng),
        lambda: test_layer_prefill_matches_bruteforce_chain(rng),
        lambda: test_kth_score_matches_stable_sort_with_ties(rng),
        lambda: test_refine_matches_bruteforce(rng, 0.6),
    ]
    caught = 0
    for p in pins:
        try:
            p()
        except AssertionError:
            caught += 1
    assert caught > 0, f"mutant {mutant} passed every pin"
