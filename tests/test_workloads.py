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
