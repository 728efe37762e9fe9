"""HostStreamedPrefill: the chunked prefill from pinned host memory, with uploads,
compute and downloads of (chunk, KV head) units on three streams, against the same
chunk loop on device-resident inputs (layer_prefill, itself checked against the
oracle in test_gpu_parity.py)."""
import numpy as np
import pytest
import torch

import sparse_attention_estimate_b200 as vsb
from sparse_attention_estimate_b200 import build as vsbuild
from tests.gpu_common import assert_gpu_outputs_close, f64
from workloads import generate_layer, small_workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    vsbuild.build()
    vsb.load_library()


# (workload, dca (C, W) or None, KV heads per unit): two chunks and two or three KV groups each
CASES = {
    "select_two_groups": (small_workload(2, seq_len=1000, chunk=512, hq=4, hkv=2, n_planted=8, kv_budget=40,
                                         ks_budget=60, refine_tau=None), None, 1),
    "refine_dca_two_groups": (small_workload(5, seq_len=1400, chunk=512, hq=10, hkv=2, n_planted=16,
                                             kv_budget=64, ks_budget=96, refine_tau=0.9), (512, 128), 1),
    "refine_three_groups_pairs": (small_workload(2, seq_len=900, chunk=384, hq=12, hkv=6, n_planted=8,
                                                 kv_budget=32, ks_budget=48, refine_tau=0.9), None, 2),
}


@pytest.mark.parametrize("name", list(CASES))
def test_streamed_from_host_matches_device_chunk_loop(name):
    w, dca, per_unit = CASES[name]
    lay = generate_layer(w)
    C, W = dca if dca else (None, None)
    cfg = vsb.Config(hq=w.hq, hkv=w.hkv, rope_base=w.rope_base, last_q=w.last_q, dca_chunk=C, dca_window=W,
                     softmax_scale=w.softmax_scale)
    q, k, v = (lay[x].cuda() for x in ("q", "k", "v"))
    ctx = vsb.Context(cfg, max_seq=w.seq_len, max_chunk=min(w.chunk, w.seq_len))
    ref = vsb.layer_prefill(ctx, q, k, v, chunk=w.chunk, kv_budget=w.kv_budget, ks_budget=w.ks_budget,
                            tau=w.refine_tau)
    assert ctx.status() == vsb.VS_OK

    sp = vsb.HostStreamedPrefill(cfg, w.seq_len, w.chunk, w.kv_budget, w.ks_budget, w.refine_tau,
                                 kv_heads_per_unit=per_unit)
    q_h, k_h, v_h = (lay[x].contiguous().pin_memory() for x in ("q", "k", "v"))
    outs = []
    for _ in range(2):  # two runs in a row: the second reuses every buffer and stream
        out_h = torch.full(tuple(lay["q"].shape), float("nan"), dtype=torch.bfloat16).pin_memory()
        sp.run(q_h, k_h, v_h, out_h)
        torch.cuda.current_stream().synchronize()
        outs.append(out_h)
    for c in sp.ctxs:
        assert c.status() == vsb.VS_OK
    assert torch.equal(outs[0], outs[1]), "two runs of the same inputs differ"
    got, want = f64(outs[0]), f64(ref)
    assert not np.isnan(got).any(), "rows left unwritten"
    for h in range(w.hq):
        assert_gpu_outputs_close(got[h], want[h], f"{name} head {h}")


def test_streamed_rejects_device_or_misshapen_buffers():
    w, _, _ = CASES["select_two_groups"]
    cfg = vsb.Config(hq=w.hq, hkv=w.hkv, rope_base=w.rope_base, softmax_scale=w.softmax_scale)
    sp = vsb.HostStreamedPrefill(cfg, w.seq_len, w.chunk, w.kv_budget, w.ks_budget, None)
    q = torch.zeros(w.hq, w.seq_len, 128, dtype=torch.bfloat16)
    kv = torch.zeros(w.hkv, w.seq_len, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        sp.run(q.cuda(), kv, kv, q.clone())  # a device tensor
    with pytest.raises(ValueError):
        sp.run(q[:, :-1], kv, kv, q.clone())  # wrong row count
    with pytest.raises(ValueError):
        vsb.HostStreamedPrefill(cfg, w.seq_len, w.chunk, 1, 1, None, kv_heads_per_unit=3)
