"""vs_select_noalloc, the selection entry point for callers that cannot
allocate device memory (for example a plugin inside an application that owns
all device memory, or a service with a fixed memory plan): it must give exactly
the sets vs_select gives, call after call, while the library allocates nothing.

This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process.
"""
import ctypes
import gc

import numpy as np
import pytest
import torch

import sparse_attention_estimate_b200 as vsb
from sparse_attention_estimate_b200 import build as vsbuild
from workloads import generate_layer, small_workload

pytestmark = pytest.mark.gpu


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def test_select_noalloc_matches_select_on_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    vsbuild.build()
    lib = vsb.load_library()
    w = small_workload(2, seq_len=4096, chunk=4096, hq=28, hkv=4, n_planted=32)
    lay = generate_layer(w)
    q, k = lay["q"].cuda(), lay["k"].cuda()
    ctx = vsb.Context(vsb.Config(hq=w.hq, hkv=w.hkv), max_seq=w.seq_len, max_chunk=w.seq_len)
    e = w.seq_len
    vert, slash, _ = ctx.estimate(q, 0, k, e)
    rng = np.random.default_rng(11)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        # different budgets per head and per call, so a stale scratch would show
        kv = torch.from_numpy(rng.integers(1, 3 * e // 2, w.hq).astype(np.int32)).cuda()
        ks = torch.from_numpy(rng.integers(1, e // 2, w.hq).astype(np.int32)).cuda()
        ref = ctx.select(vert, slash, e, kv, ks)
        got = [torch.full((w.hq, e), -1, dtype=torch.int32, device="cuda"),
               torch.full((w.hq,), -1, dtype=torch.int32, device="cuda"),
               torch.full((w.hq, e), -1, dtype=torch.int32, device="cuda"),
               torch.full((w.hq,), -1, dtype=torch.int32, device="cuda")]
        # nothing may be allocated by a call: neither through torch nor on the device.
        # The first call on a device does the one-time set-up (the address lookup, at
        # which CUDA's lazy module loading may reserve the static array), so the device
        # check applies from the second call on. Garbage collection is held off so
        # earlier tests' tensors are not freed meanwhile.
        gc.collect()
        gc.disable()
        try:
            torch.cuda.synchronize()
            n0, free0 = torch.cuda.memory_allocated(), torch.cuda.mem_get_info()[0]
            st = lib.vs_select_noalloc(w.hq, _p(vert), _p(slash), vert.stride(0), e, _p(kv), _p(ks), _p(got[0]),
                                       e, _p(got[1]), _p(got[2]), e, _p(got[3]), stream)
            assert st == vsb.VS_OK, lib.vs_last_error()
            torch.cuda.synchronize()
            assert torch.cuda.memory_allocated() == n0
            if call > 0:
                assert torch.cuda.mem_get_info()[0] == free0
        finally:
            gc.enable()
        assert ctx.status() == vsb.VS_OK
        r_vi, r_vc, r_so, r_sc = [t.cpu() for t in ref]
        g_vi, g_vc, g_so, g_sc = [t.cpu() for t in got]
        assert torch.equal(g_vc, r_vc) and torch.equal(g_sc, r_sc), call
        for h in range(w.hq):
            assert torch.equal(g_vi[h, : r_vc[h]], r_vi[h, : r_vc[h]]), (call, h)
            assert torch.equal(g_so[h, : r_sc[h]], r_so[h, : r_sc[h]]), (call, h)
        assert int(r_vc.min()) >= 1 and int(r_sc.min()) >= 1


def test_select_noalloc_rejects_sizes_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    vsbuild.build()
    lib = vsb.load_library()
    e = 1 << 20
    dummy = torch.empty(16, dtype=torch.int32, device="cuda")
    p = _p(dummy)
    st = lib.vs_select_noalloc(40, p, p, e, e, p, p, p, e, p, p, e, p, None)  # 40 heads x 1M: 80 MiB
    assert st == vsb.VS_ERR_UNSUPPORTED
    assert b"no-alloc scratch" in lib.vs_last_error()
    st = lib.vs_select_noalloc(4, p, p, 4096, 4096, p, p, p, 100, p, p, 4096, p, None)  # cap below e
    assert st == vsb.VS_ERR_INVALID_ARG
