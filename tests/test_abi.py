"""The C ABI on a machine without a GPU: the library builds, loads, exports every
function include/vs.h declares, and rejects bad arguments on the host."""
import ctypes
import os
import re

import pytest

import sparse_attention_estimate_b200 as vsb
from sparse_attention_estimate_b200 import build as vsbuild

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "vs.h")


@pytest.fixture(scope="module")
def lib():
    vsbuild.build()
    return vsb.load_library()


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*VS_API\s+(?:const\s+)?\w+\s*\*?\s*(\w+)\s*\(", src, flags=re.M)))


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert "vs_sparse_prefill" in names and "dca_remap" in names and len(names) >= 14
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(vsb.EXPORTS)


def _cfg(**kw):
    c = vsb.Config(hq=kw.pop("hq", 28), hkv=kw.pop("hkv", 4), **kw).to_c()
    return c


def test_workspace_size_and_validation(lib):
    n = ctypes.c_size_t(0)
    c = _cfg()
    assert lib.vs_workspace_size(ctypes.byref(c), 32768, 32768, ctypes.byref(n)) == vsb.VS_OK
    assert n.value > 28 * 32768 * 128 * 2  # at least the rotated query buffer
    c5 = _cfg(hq=40, hkv=8, dca_chunk=262144)
    m = ctypes.c_size_t(0)
    assert lib.vs_workspace_size(ctypes.byref(c5), 1 << 20, 32768, ctypes.byref(m)) == vsb.VS_OK
    assert m.value > 2 * 8 * (1 << 20) * 256  # two rotated key caches with DCA
    bad = _cfg()
    bad.head_dim = 64
    assert lib.vs_workspace_size(ctypes.byref(bad), 1024, 1024, ctypes.byref(n)) == vsb.VS_ERR_UNSUPPORTED
    assert b"128" in lib.vs_last_error()
    bad = _cfg(hq=28, hkv=5)
    assert lib.vs_workspace_size(ctypes.byref(bad), 1024, 1024, ctypes.byref(n)) == vsb.VS_ERR_UNSUPPORTED
    bad = _cfg(hq=40, hkv=4)  # group of 10 > 8
    assert lib.vs_workspace_size(ctypes.byref(bad), 1024, 1024, ctypes.byref(n)) == vsb.VS_ERR_UNSUPPORTED
    bad = _cfg(dca_chunk=1000)  # not a multiple of 128
    assert lib.vs_workspace_size(ctypes.byref(bad), 1024, 1024, ctypes.byref(n)) == vsb.VS_ERR_UNSUPPORTED
    bad = _cfg(last_q=65)
    assert lib.vs_workspace_size(ctypes.byref(bad), 1024, 1024, ctypes.byref(n)) == vsb.VS_ERR_INVALID_ARG
    assert lib.vs_workspace_size(ctypes.byref(c), 1024, 2048, ctypes.byref(n)) == vsb.VS_ERR_INVALID_ARG
    assert lib.vs_workspace_size(None, 1024, 1024, ctypes.byref(n)) == vsb.VS_ERR_INVALID_ARG


def test_context_create_rejects_missing_workspace(lib):
    c = _cfg()
    h = ctypes.c_void_p()
    assert lib.vs_context_create(ctypes.byref(c), 1024, 1024, None, 0, None, ctypes.byref(h)) == vsb.VS_ERR_WORKSPACE
    assert lib.vs_context_create(ctypes.byref(c), 1024, 1024, ctypes.c_void_p(0x1001), 1 << 30, None,
                                 ctypes.byref(h)) == vsb.VS_ERR_WORKSPACE  # misaligned
    assert lib.vs_context_create(ctypes.byref(c), 1024, 1024, ctypes.c_void_p(0x100000), 16, None,
                                 ctypes.byref(h)) == vsb.VS_ERR_WORKSPACE  # too small


def test_calls_reject_null_context(lib):
    assert lib.vs_estimate(None, None, 0, 0, None, 0, 0, None, None, 0, None, None) == vsb.VS_ERR_INVALID_ARG
    assert lib.vs_select(None, None, None, 0, 0, None, None, None, 0, None, None, 0, None, None) == vsb.VS_ERR_INVALID_ARG
    assert lib.vs_sparse_prefill(None, None, 0, 0, 0, None, None, 0, None, 0, None, None, 0, None, None, None,
                                 None) == vsb.VS_ERR_INVALID_ARG
    assert lib.vs_context_reset(None) == vsb.VS_ERR_INVALID_ARG
    assert lib.vs_set_wait_limit(None, 10 ** 9) == vsb.VS_ERR_INVALID_ARG
    assert lib.vs_set_deterministic(None, 1) == vsb.VS_ERR_INVALID_ARG


@pytest.mark.skipif(__import__("torch").cuda.is_available(), reason="checks the behaviour without a CUDA device")
def test_python_entry_points_fail_loudly_without_a_gpu():
    """No CPU fallback: without a CUDA device every entry point of the binding raises
    before doing any work (the oracle is test infrastructure, never a product path)."""
    cfg = vsb.Config(hq=2, hkv=1)
    with pytest.raises(RuntimeError, match="CUDA"):
        vsb.Context(cfg, max_seq=256, max_chunk=256)
    with pytest.raises(RuntimeError, match="CUDA"):
        vsb.HostStreamedPrefill(cfg, 256, 256, 8, 8, None)
