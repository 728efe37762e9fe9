"""Python binding of the sm_100a sparse-prefill library (libvs.so).

The library implements, for one GQA attention layer, the chunked prefill of the
Qwen2.5-1M inference framework (0h-n0.github.io explainer of the Qwen2.5-1M
report: "Sparse Attention", "Chunked Prefill", "Sparsity Refinement", "Length
Extrapolation" / DCA, and the sparse_attention_with_dca chunk loop of
"Algorithm"). Every step runs in the library's CUDA kernels; this module only
marshals torch tensors (device memory, the current stream) into the C ABI of
include/vs.h. There is no CPU fallback: without the built library or a CUDA
device the calls raise.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# the in-tree build; VS_LIBRARY may name another build of the same library
LIB_PATH = os.environ.get("VS_LIBRARY") or os.path.join(_PKG, "libvs.so")

VS_OK, VS_ERR_INVALID_ARG, VS_ERR_UNSUPPORTED, VS_ERR_WORKSPACE = 0, 1, 2, 3
VS_ERR_CUDA, VS_ERR_TIMEOUT, VS_ERR_DEVICE_CHECK = 4, 5, 6
STATUS_NAMES = {0: "VS_OK", 1: "VS_ERR_INVALID_ARG", 2: "VS_ERR_UNSUPPORTED", 3: "VS_ERR_WORKSPACE",
                4: "VS_ERR_CUDA", 5: "VS_ERR_TIMEOUT", 6: "VS_ERR_DEVICE_CHECK"}

EXPORTS = ("vs_workspace_size", "vs_context_create", "vs_context_destroy", "vs_context_reset",
           "vs_set_wait_limit", "dca_remap", "vs_estimate", "vs_select", "vs_refine",
           "vs_sparse_prefill", "vs_prefill_stats", "vs_status_poll", "vs_selftest_wait_timeout",
           "vs_last_error", "vs_set_prefill_events", "vs_kernel_launches", "vs_select_noalloc",
           "vs_calibrate_accumulate", "vs_set_deterministic")


class VsError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class AttnCfg(ctypes.Structure):
    _fields_ = [("hq", ctypes.c_int32), ("hkv", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("last_q", ctypes.c_int32), ("softmax_scale", ctypes.c_float),
                ("rope_base", ctypes.c_double), ("dca_enabled", ctypes.c_int32),
                ("dca_chunk_size", ctypes.c_int64), ("dca_local_window", ctypes.c_int64),
                ("refine_dca_positions", ctypes.c_int32)]


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads libvs.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m sparse_attention_estimate_b200.build`")
    lib = ctypes.CDLL(path)
    P, I32, I64, F32, U64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_uint64
    sig = {
        "vs_workspace_size": [ctypes.POINTER(AttnCfg), I64, I64, ctypes.POINTER(ctypes.c_size_t)],
        "vs_context_create": [ctypes.POINTER(AttnCfg), I64, I64, P, ctypes.c_size_t, P, ctypes.POINTER(P)],
        "vs_context_destroy": [P],
        "vs_context_reset": [P],
        "vs_set_wait_limit": [P, U64],
        "vs_set_deterministic": [P, I32],
        "dca_remap": [P, I64, I64, P, P, P, P, P],
        "vs_estimate": [P, P, I64, I64, P, I64, I64, P, P, I64, P, P],
        "vs_select": [P, P, P, I64, I64, P, P, P, I32, P, P, I32, P, P],
        "vs_refine": [P, P, I64, I64, P, I64, I64, P, P, I64, P, F32, I32, P, P, P, I32, P, P, I32, P, P, P],
        "vs_sparse_prefill": [P, P, I64, I64, I64, P, P, I64, P, I32, P, P, I32, P, P, P, P],
        "vs_prefill_stats": [P, P, ctypes.POINTER(I64)],
        "vs_status_poll": [P, P],
        "vs_selftest_wait_timeout": [P, U64, P],
        "vs_set_prefill_events": [P, P, P],
        "vs_select_noalloc": [I32, P, P, I64, I64, P, P, P, I32, P, P, I32, P, P],
        "vs_calibrate_accumulate": [P, P, P, P, P, P],
    }
    for name, args in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = ctypes.c_int
    lib.vs_kernel_launches.argtypes = []
    lib.vs_kernel_launches.restype = ctypes.c_uint64
    lib.vs_last_error.argtypes = []
    lib.vs_last_error.restype = ctypes.c_char_p
    _lib = lib
    return lib


def _check(status: int) -> None:
    if status != VS_OK:
        raise VsError(status, load_library().vs_last_error().decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _rows(t: torch.Tensor, r0: int):
    """Pointer to row r0 of every head of a [heads, rows, d] tensor (the head
    stride stays t.shape[1] rows): a zero-copy view of rows r0.. ."""
    return ctypes.c_void_p(t.data_ptr() + r0 * t.stride(1) * t.element_size())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _bf16_3d(t: torch.Tensor, name: str) -> torch.Tensor:
    if t.dtype != torch.bfloat16 or t.dim() != 3 or t.shape[-1] != 128 or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA bf16 tensor [heads, rows, 128]")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


@dataclass
class Config:
    hq: int
    hkv: int
    rope_base: float = 1.0e7
    softmax_scale: Optional[float] = None
    last_q: int = 64
    dca_chunk: Optional[int] = None
    dca_window: Optional[int] = None
    refine_dca_positions: bool = False  # recall at DCA positions (DCA only)

    def to_c(self) -> AttnCfg:
        c = AttnCfg()
        c.hq, c.hkv, c.head_dim, c.last_q = self.hq, self.hkv, 128, self.last_q
        c.softmax_scale = self.softmax_scale if self.softmax_scale is not None else 1.0 / math.sqrt(128)
        c.rope_base = self.rope_base
        c.dca_enabled = 1 if self.dca_chunk else 0
        c.dca_chunk_size = self.dca_chunk or 0
        c.dca_local_window = (self.dca_window if self.dca_window is not None else
                              (self.dca_chunk // 32 if self.dca_chunk else 0))
        c.refine_dca_positions = 1 if self.refine_dca_positions else 0
        return c


def kernel_launches() -> int:
    """Kernels the library has launched in this process."""
    return int(load_library().vs_kernel_launches())


def workspace_size(cfg: Config, max_seq: int, max_chunk: int) -> int:
    n = ctypes.c_size_t(0)
    c = cfg.to_c()
    _check(load_library().vs_workspace_size(ctypes.byref(c), max_seq, max_chunk, ctypes.byref(n)))
    return n.value


class Context:
    """A library context over a torch-allocated device workspace."""

    def __init__(self, cfg: Config, max_seq: int, max_chunk: int, device=None,
                 workspace: Optional[torch.Tensor] = None):
        if not torch.cuda.is_available():
            raise RuntimeError("the sparse-prefill library needs a CUDA device")
        self.lib = load_library()
        self.cfg = cfg
        self.max_seq, self.max_chunk = max_seq, max_chunk
        self.device = torch.device(device or "cuda")
        nbytes = workspace_size(cfg, max_seq, max_chunk)
        if workspace is None:
            workspace = torch.empty(nbytes + 256, dtype=torch.uint8, device=self.device)
        self._ws = workspace
        base = workspace.data_ptr()
        off = (-base) % 256
        self._ws_ptr = base + off
        self._ws_bytes = workspace.numel() - off
        self._c_cfg = cfg.to_c()
        h = ctypes.c_void_p()
        with torch.cuda.device(self.device):
            _check(self.lib.vs_context_create(ctypes.byref(self._c_cfg), max_seq, max_chunk,
                                              ctypes.c_void_p(self._ws_ptr), self._ws_bytes, _stream(),
                                              ctypes.byref(h)))
        self.handle = h

    def close(self):
        if getattr(self, "handle", None):
            self.lib.vs_context_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # ------------------------------------------------------------------ calls
    def reset(self):
        _check(self.lib.vs_context_reset(self.handle))

    def set_wait_limit(self, ns: int):
        _check(self.lib.vs_set_wait_limit(self.handle, ns))

    def set_deterministic(self, on: bool):
        """Bitwise reproducible prefill (every work list swept from its start)."""
        _check(self.lib.vs_set_deterministic(self.handle, 1 if on else 0))

    def status(self) -> int:
        """Synchronises and returns (and clears) the device error word status."""
        return self.lib.vs_status_poll(self.handle, _stream())

    def dca_remap(self, pos0: int, n: int):
        out = [torch.empty(n, dtype=torch.int32, device=self.device) for _ in range(4)]
        _check(self.lib.dca_remap(self.handle, pos0, n, *[_ptr(t) for t in out], _stream()))
        return tuple(out)

    def estimate(self, q: torch.Tensor, q_pos0: int, k: torch.Tensor, e: int, out=None, full=False):
        """vert [hq, e], slash [hq, e], lse [hq, 64] for the chunk [q_pos0, e).
        q's row 0 holds position q_pos0, or position 0 when full=True (then q is
        the whole sequence and the chunk is a zero-copy row view of it)."""
        _bf16_3d(q, "q"), _bf16_3d(k, "k")
        hq = self.cfg.hq
        if out is None:
            vert = torch.empty(hq, e, dtype=torch.float32, device=self.device)
            slash = torch.empty(hq, e, dtype=torch.float32, device=self.device)
            lse = torch.empty(hq, 64, dtype=torch.float32, device=self.device)
        else:
            vert, slash, lse = out
        qp = _rows(q, q_pos0) if full else _ptr(q)
        _check(self.lib.vs_estimate(self.handle, qp, q.shape[1], q_pos0, _ptr(k), k.shape[1], e,
                                    _ptr(vert), _ptr(slash), vert.stride(0), _ptr(lse), _stream()))
        return vert, slash, lse

    def _sets(self, cap_v, cap_s):
        hq = self.cfg.hq
        d = self.device
        return (torch.empty(hq, cap_v, dtype=torch.int32, device=d), torch.empty(hq, dtype=torch.int32, device=d),
                torch.empty(hq, cap_s, dtype=torch.int32, device=d), torch.empty(hq, dtype=torch.int32, device=d))

    def select(self, vert, slash, e: int, kv_budget, ks_budget, cap_v=None, cap_s=None, sets=None):
        cap_v = cap_v or e
        cap_s = cap_s or e
        v_idx, v_cnt, s_off, s_cnt = sets if sets is not None else self._sets(cap_v, cap_s)
        _check(self.lib.vs_select(self.handle, _ptr(vert), _ptr(slash), vert.stride(0), e, _ptr(kv_budget),
                                  _ptr(ks_budget), _ptr(v_idx), v_idx.shape[1], _ptr(v_cnt), _ptr(s_off),
                                  s_off.shape[1], _ptr(s_cnt), _stream()))
        return v_idx, v_cnt, s_off, s_cnt

    def refine(self, q, q_pos0, k, e, vert, slash, lse, tau, kv_budget, ks_budget, max_iters=19,
               cap_v=None, cap_s=None, sets=None, recall=None, full=False):
        """kv_budget / ks_budget (int32 [hq] on the device) are updated in place."""
        cap_v = cap_v or e
        cap_s = cap_s or e
        v_idx, v_cnt, s_off, s_cnt = sets if sets is not None else self._sets(cap_v, cap_s)
        if recall is None:
            recall = torch.empty(self.cfg.hq, dtype=torch.float32, device=self.device)
        qp = _rows(q, q_pos0) if full else _ptr(q)
        _check(self.lib.vs_refine(self.handle, qp, q.shape[1], q_pos0, _ptr(k), k.shape[1], e, _ptr(vert),
                                  _ptr(slash), vert.stride(0), _ptr(lse), float(tau), int(max_iters),
                                  _ptr(kv_budget), _ptr(ks_budget), _ptr(v_idx), v_idx.shape[1], _ptr(v_cnt),
                                  _ptr(s_off), s_off.shape[1], _ptr(s_cnt), _ptr(recall), _stream()))
        return (v_idx, v_cnt, s_off, s_cnt), recall

    def sparse_prefill(self, q, q_pos0: int, e: int, k, v, sets, out=None, lse=None, want_lse=True,
                       full=False):
        """Rows [q_pos0, e) of the chunk. q, out: [hq, rows, 128] (row 0 = position
        q_pos0, or position 0 with full=True); lse: [hq, rows] like out."""
        _bf16_3d(q, "q"), _bf16_3d(k, "k"), _bf16_3d(v, "v")
        v_idx, v_cnt, s_off, s_cnt = sets
        if out is None:
            out = torch.empty_like(q)
        if lse is None and want_lse:
            lse = torch.empty(q.shape[0], q.shape[1], dtype=torch.float32, device=self.device)
        if out.shape != q.shape or (lse is not None and tuple(lse.shape) != tuple(q.shape[:2])):
            raise ValueError("out must match q and lse must be [hq, rows]")
        r0 = q_pos0 if full else 0
        lp = None if lse is None else ctypes.c_void_p(lse.data_ptr() + r0 * lse.stride(1) * 4)
        _check(self.lib.vs_sparse_prefill(self.handle, _rows(q, r0), q.shape[1], q_pos0, e, _ptr(k), _ptr(v),
                                          k.shape[1], _ptr(v_idx), v_idx.shape[1], _ptr(v_cnt), _ptr(s_off),
                                          s_off.shape[1], _ptr(s_cnt), _rows(out, r0), lp, _stream()))
        return out, lse

    def prefill_stats(self):
        a = (ctypes.c_int64 * 2)()
        _check(self.lib.vs_prefill_stats(self.handle, _stream(), a))
        return int(a[0]), int(a[1])

    def set_prefill_events(self, start: Optional[torch.cuda.Event], stop: Optional[torch.cuda.Event]):
        """Record `start`/`stop` around the attention kernel of each following
        sparse_prefill (None, None to stop). The events must already exist
        (record them once before passing them)."""
        a = None if start is None else ctypes.c_void_p(start.cuda_event)
        b = None if stop is None else ctypes.c_void_p(stop.cuda_event)
        _check(self.lib.vs_set_prefill_events(self.handle, a, b))

    def calibrate_accumulate(self, kv_budget, ks_budget, kv_acc, ks_acc):
        """kv_acc / ks_acc (int32 [hq] on the device) keep the larger budgets, in place."""
        _check(self.lib.vs_calibrate_accumulate(self.handle, _ptr(kv_budget), _ptr(ks_budget), _ptr(kv_acc),
                                                _ptr(ks_acc), _stream()))

    def selftest_wait_timeout(self, limit_ns: int):
        _check(self.lib.vs_selftest_wait_timeout(self.handle, limit_ns, _stream()))


def calibrate(ctx: Context, q: torch.Tensor, k: torch.Tensor, *, chunk: int, kv_budget: int, ks_budget: int,
              tau: float, max_iters: int = 19):
    """Offline form of sparsity refinement (explainer, Chunked Prefill: the budgets
    are improved once on a calibration sequence): every chunk of the calibration
    sequence q, k is estimated and refined from the base budgets, and each head keeps
    the largest refined budgets over the chunks. Returns (kv, ks), int32 [hq] on the
    device, for layer_prefill(..., kv_budget=kv, ks_budget=ks, tau=None)."""
    hq, n = q.shape[0], q.shape[1]
    dev = q.device
    kv_c = torch.zeros(hq, dtype=torch.int32, device=dev)
    ks_c = torch.zeros(hq, dtype=torch.int32, device=dev)
    for cs in range(0, n, chunk):
        e = min(cs + chunk, n)
        vert, slash, lse = ctx.estimate(q, cs, k, e, full=True)
        kvb = torch.full((hq,), kv_budget, dtype=torch.int32, device=dev)
        ksb = torch.full((hq,), ks_budget, dtype=torch.int32, device=dev)
        ctx.refine(q, cs, k, e, vert, slash, lse, tau, kvb, ksb, max_iters=max_iters, full=True)
        ctx.calibrate_accumulate(kvb, ksb, kv_c, ks_c)
    return kv_c, ks_c


def layer_prefill(ctx: Context, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, chunk: int,
                  kv_budget, ks_budget, tau: Optional[float], out: Optional[torch.Tensor] = None,
                  max_iters: int = 19, keep=None):
    """The chunk loop of sparse_attention_with_dca (explainer, "Algorithm"): for
    each chunk [cs, e) of `chunk` queries, estimate with the chunk's last queries,
    select (and refine when tau is given), then attend the chunk's rows over keys
    [0, e). q: [hq, N, 128]; k, v: [hkv, N, 128] (the KV cache, rows at their
    positions). kv_budget / ks_budget: ints for every head, or int32 [hq] device
    tensors (per-head budgets, e.g. from calibrate). Returns the output
    [hq, N, 128] and, when `keep` is a list, appends per-chunk intermediates to it."""
    hq, n = q.shape[0], q.shape[1]
    dev = q.device
    if out is None:
        out = torch.empty_like(q)
    def per_head(b):
        if isinstance(b, torch.Tensor):
            return b.to(device=dev, dtype=torch.int32)
        return torch.full((hq,), int(b), dtype=torch.int32, device=dev)

    base_v, base_s = per_head(kv_budget), per_head(ks_budget)
    lse_o = torch.empty(hq, n, dtype=torch.float32, device=dev)
    for cs in range(0, n, chunk):
        e = min(cs + chunk, n)
        vert, slash, lse = ctx.estimate(q, cs, k, e, full=True)
        kvb, ksb = base_v.clone(), base_s.clone()
        if tau is None:
            sets = ctx.select(vert, slash, e, kvb, ksb)
            recall = None
        else:
            sets, recall = ctx.refine(q, cs, k, e, vert, slash, lse, tau, kvb, ksb, max_iters=max_iters,
                                      full=True)
        ctx.sparse_prefill(q, cs, e, k, v, sets, out=out, lse=lse_o, full=True)
        if keep is not None:
            keep.append(dict(cs=cs, e=e, vert=vert, slash=slash, lse_est=lse, kv=kvb, ks=ksb, sets=sets,
                             recall=recall, lse=lse_o[:, cs:e], out=out[:, cs:e]))
    return out


class HostStreamedPrefill:
    """layer_prefill from pinned host memory, with the copies overlapped.

    For a caller whose Q, K, V live in host memory and who wants O back there. The
    work is cut into units of (chunk, KV-head group): no step of the path mixes KV
    groups, and chunk c only needs the KV rows of chunks <= c. Each unit uploads its
    new rows (the chunk's query rows of the group's heads, the chunk's K and V rows
    of its KV heads) on an upload stream, computes estimate -> refine/select ->
    sparse prefill on the caller's current stream with one library context per group,
    and downloads its output rows on a download stream, so unit u's upload and unit
    u-1's download run while unit u-1 computes. Results equal layer_prefill up to
    rounding: a context over fewer KV heads splits the estimation's key range into
    more parts, which changes the order of the partial sums.

    Device buffers and contexts are allocated here, once; run() allocates nothing on
    the device. kv_budget / ks_budget: ints or int32 [hq] tensors (e.g. calibrated)."""

    def __init__(self, cfg: Config, seq_len: int, chunk: int, kv_budget, ks_budget, tau: Optional[float],
                 max_iters: int = 19, kv_heads_per_unit: int = 1, device=None):
        from dataclasses import replace

        if cfg.hkv % kv_heads_per_unit:
            raise ValueError("kv_heads_per_unit must divide hkv")
        self.device = torch.device(device or "cuda")
        dev = self.device
        self.cfg, self.n, self.chunk, self.tau, self.max_iters = cfg, seq_len, chunk, tau, max_iters
        g = cfg.hq // cfg.hkv
        self.groups = [(k0, k0 + kv_heads_per_unit) for k0 in range(0, cfg.hkv, kv_heads_per_unit)]
        hq_u = g * kv_heads_per_unit
        self.ctxs = [Context(replace(cfg, hq=hq_u, hkv=kv_heads_per_unit), max_seq=seq_len,
                             max_chunk=min(chunk, seq_len), device=dev) for _ in self.groups]
        bf = torch.bfloat16
        self.q = torch.empty(cfg.hq, seq_len, 128, dtype=bf, device=dev)
        self.k = torch.empty(cfg.hkv, seq_len, 128, dtype=bf, device=dev)
        self.v = torch.empty(cfg.hkv, seq_len, 128, dtype=bf, device=dev)
        self.out = torch.empty_like(self.q)
        self.lse = torch.empty(cfg.hq, seq_len, dtype=torch.float32, device=dev)

        def per_head(b):
            if isinstance(b, torch.Tensor):
                return b.to(device=dev, dtype=torch.int32)
            return torch.full((cfg.hq,), int(b), dtype=torch.int32, device=dev)

        self.base_v, self.base_s = per_head(kv_budget), per_head(ks_budget)
        f32, i32 = torch.float32, torch.int32
        self.bufs = []
        for _ in self.groups:
            self.bufs.append(dict(
                vert=torch.empty(hq_u, seq_len, dtype=f32, device=dev),
                slash=torch.empty(hq_u, seq_len, dtype=f32, device=dev),
                lse_est=torch.empty(hq_u, 64, dtype=f32, device=dev),
                kv=torch.empty(hq_u, dtype=i32, device=dev), ks=torch.empty(hq_u, dtype=i32, device=dev),
                recall=torch.empty(hq_u, dtype=f32, device=dev),
                sets=(torch.empty(hq_u, seq_len, dtype=i32, device=dev), torch.empty(hq_u, dtype=i32, device=dev),
                      torch.empty(hq_u, seq_len, dtype=i32, device=dev), torch.empty(hq_u, dtype=i32, device=dev))))
        self.up = torch.cuda.Stream(device=dev)
        self.down = torch.cuda.Stream(device=dev)
        self.g = g

    def run(self, q_h: torch.Tensor, k_h: torch.Tensor, v_h: torch.Tensor, out_h: torch.Tensor) -> None:
        """q_h, out_h: [hq, N, 128]; k_h, v_h: [hkv, N, 128]; bf16, pinned host memory.
        Asynchronous on the current stream: out_h is complete once it has synchronised."""
        cfg, g = self.cfg, self.g
        for t, shape in ((q_h, self.q.shape), (k_h, self.k.shape), (v_h, self.v.shape), (out_h, self.out.shape)):
            if t.is_cuda or t.dtype != torch.bfloat16 or tuple(t.shape) != tuple(shape) or not t.is_contiguous():
                raise ValueError("host tensors must be contiguous bf16 [heads, N, 128] in host memory")
        cur = torch.cuda.current_stream(self.device)
        self.up.wait_stream(cur)    # the previous run's compute has read the device inputs
        self.down.wait_stream(cur)
        for ctx in self.ctxs:
            ctx.reset()
        for cs in range(0, self.n, self.chunk):
            e = min(cs + self.chunk, self.n)
            for ui, (k0, k1) in enumerate(self.groups):
                h0, h1 = k0 * g, k1 * g
                with torch.cuda.stream(self.up):
                    for h in range(h0, h1):
                        self.q[h, cs:e].copy_(q_h[h, cs:e], non_blocking=True)
                    for h in range(k0, k1):
                        self.k[h, cs:e].copy_(k_h[h, cs:e], non_blocking=True)
                        self.v[h, cs:e].copy_(v_h[h, cs:e], non_blocking=True)
                    ready = torch.cuda.Event()
                    ready.record(self.up)
                cur.wait_event(ready)
                ctx, b = self.ctxs[ui], self.bufs[ui]
                q, k, v = self.q[h0:h1], self.k[k0:k1], self.v[k0:k1]
                vert, slash = b["vert"][:, :e], b["slash"][:, :e]
                ctx.estimate(q, cs, k, e, out=(vert, slash, b["lse_est"]), full=True)
                b["kv"].copy_(self.base_v[h0:h1])
                b["ks"].copy_(self.base_s[h0:h1])
                if self.tau is None:
                    ctx.select(vert, slash, e, b["kv"], b["ks"], sets=b["sets"])
                else:
                    ctx.refine(q, cs, k, e, vert, slash, b["lse_est"], self.tau, b["kv"], b["ks"],
                               max_iters=self.max_iters, sets=b["sets"], recall=b["recall"], full=True)
                ctx.sparse_prefill(q, cs, e, k, v, b["sets"], out=self.out[h0:h1], lse=self.lse[h0:h1], full=True)
                done = torch.cuda.Event()
                done.record(cur)
                with torch.cuda.stream(self.down):
                    self.down.wait_event(done)
                    for h in range(h0, h1):
                        out_h[h, cs:e].copy_(self.out[h, cs:e], non_blocking=True)
        cur.wait_stream(self.down)
