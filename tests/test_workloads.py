"""The seeded generator: determinism, row subsets, structure (CPU only)."""
import torch

from workloads import WORKLOADS, generate_head, planted_positions, small_workload, structure


def test_generator_is_deterministic_and_rows_are_bit_identical():
    w = small_workload(2, seq_len=1000, chunk=512, hq=4, hkv=2)
    a = generate_head(w, "q", 3)
    b = generate_head(w, "q", 3)
    assert torch.equal(a, b) and a.dtype == torch.bfloat16 and a.shape == (1000, 128)
    rows = torch.tensor([0, 5, 999, 640])
    assert torch.equal(generate_head(w, "q", 3, rows=rows), a[rows])
    k = generate_head(w, "k", 1)
    assert torch.equal(generate_head(w, "k", 1, rows=rows), k[rows])
    assert not torch.equal(generate_head(w, "k", 0), k)


def test_structure_vectors():
    w = small_workload(1, seq_len=4096, chunk=4096)
    st = structure(w)
    u, z = st["u"], st["z"]
    assert abs(float(u.norm()) - 1) < 1e-6
    assert torch.count_nonzero(u[:60]) == 0 and torch.count_nonzero(u[64:124]) == 0
    assert z.shape == (64, 128) and torch.allclose(z.norm(dim=1), torch.ones(64))
    p = planted_positions(w)
    assert len(p) == 16 and torch.all(p[1:] > p[:-1])


def test_workload_table():
    assert [WORKLOADS[i].seq_len for i in range(1, 6)] == [4096, 32768, 131072, 262144, 1048576]
    assert WORKLOADS[4].dca_window == 2048 and WORKLOADS[4].dca_stride == 63488
    assert WORKLOADS[5].dca_window == 8192 and WORKLOADS[5].dca_stride == 253952
    assert WORKLOADS[5].n_chunks == 32 and WORKLOADS[3].chunk_bounds(3) == (98304, 131072)


def test_peaked_variant_scales_only_the_random_part_of_q():
    """q_scale multiplies Q's N(0,1) draw before the structure is added: the
    difference to the unscaled head is (q_scale - 1) times that draw, K and V are
    untouched, and base scaled logits of distant pairs have std near q_scale."""
    import math

    w1 = small_workload(2, seq_len=2048, chunk=2048, hq=2, hkv=1)
    w4 = small_workload(6, seq_len=2048, chunk=2048, hq=2, hkv=1)
    assert w4.q_scale == 4.0 and w1.q_scale == 1.0 and w4.seed == w1.seed
    assert torch.equal(generate_head(w1, "k", 0), generate_head(w4, "k", 0))
    assert torch.equal(generate_head(w1, "v", 0), generate_head(w4, "v", 0))
    from workloads.gen import _gen

    base = torch.randn(2048, 128, generator=_gen(w1.seed, "q", 1))
    d = generate_head(w4, "q", 1).float() - generate_head(w1, "q", 1).float()
    assert torch.allclose(d, 3.0 * base, atol=0.1, rtol=0.02)
    q, k = generate_head(w4, "q", 0).float(), generate_head(w4, "k", 0).float()
    gen = torch.Generator().manual_seed(0)
    i = torch.randint(0, 2048, (4000,), generator=gen)
    j = torch.randint(0, 2048, (4000,), generator=gen)
    far = (i - j).abs() >= 128
    lg = (q[i] * k[j]).sum(1) / math.sqrt(128)
    assert 3.6 < float(lg[far].std()) < 4.8


def test_yarn_temperature():
    """sqrt(1/t) = 0.1 ln(s) + 1 with s = N / training length (explainer, Length
    Extrapolation): at 1M over 262,144 tokens, s = 4; no scaling for s <= 1."""
    import math

    w = WORKLOADS[8]
    assert w.yarn_train_len == 262144 and w.seq_len == 4 * 262144
    assert math.isclose(math.sqrt(w.yarn_factor), 0.1 * math.log(4.0) + 1.0, rel_tol=1e-15)
    assert math.isclose(w.softmax_scale, w.yarn_factor / math.sqrt(128), rel_tol=1e-15)
    assert WORKLOADS[5].yarn_factor == 1.0 and WORKLOADS[5].softmax_scale == 1 / math.sqrt(128)
    short = small_workload(8, seq_len=1000, chunk=512, yarn_train_len=4096)
    assert short.yarn_factor == 1.0


def test_planted_columns_stand_out_in_the_oracle_estimate():
    """Workload sanity (not parity), on the 4096-token workload: the planted key columns
    collect clearly more estimation mass than the other columns. Their boost is
    K += 4u, Q += 1.5u, i.e. +6 raw, +0.53 scaled logits (x1.7 probability), which
    puts every planted column above the median column but not all of them inside a
    256-column budget: 8 of 16 make it on head 0 (the rest rank up to ~1500)."""
    import numpy as np

    import oracle.vs_oracle as vo
    from workloads import WORKLOADS, generate_layer, structure

    w = WORKLOADS[1]
    planted = np.asarray(structure(w)["planted"])
    lay = generate_layer(w)
    q = lay["q"].float().double().numpy()
    k = lay["k"].float().double().numpy()
    e, nr = w.seq_len, w.last_q
    others = np.setdiff1d(np.arange(e - 128), planted)  # outside the band of the estimation rows
    for h in range(w.hq):
        _, vert, _, _ = vo.estimate(q[h, e - nr:e], k[h // w.group], e, w.rope_base, w.softmax_scale)
        assert vert[planted].mean() >= 2.0 * vert[others].mean(), h
        rank = np.argsort(np.argsort(-vert, kind="stable"), kind="stable")
        assert rank[planted].max() < e // 2, h
