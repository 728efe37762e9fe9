"""The five synthetic single-layer workloads and small variants of them.

Shapes follow the Qwen2.5-1M report explainer (0h-n0.github.io, "Inference
framework" / "Chunked Prefill": 32,768-token chunks, last 64 queries of each
chunk drive selection; Table 2: final RoPE base 10,000,000) and the two model
shapes: Qwen2.5-7B (28 query / 4 KV heads, head_dim 128) and a 14B-shaped layer
(40 / 8). DCA constants: chunk size C as given per workload, local window
W = C / 32, stride S = C - W (a reading: the pages fix C and the three rules only).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace
from typing import Optional


@dataclass(frozen=True)
class Workload:
    name: str
    hq: int
    hkv: int
    seq_len: int
    seed: int
    n_planted: int
    kv_budget: int  # base vertical budget k_v
    ks_budget: int  # base slash budget k_s
    refine_tau: Optional[float]  # None: no refinement
    dca_chunk: Optional[int] = None  # DCA chunk size C (None: continuous RoPE)
    chunk: int = 32768  # prefill chunk length
    head_dim: int = 128
    rope_base: float = 1.0e7
    last_q: int = 64
    # Sparse-regime variant: the N(0, 1) part of Q is multiplied by q_scale, so the
    # base scaled logits q.k / sqrt(D) have standard deviation q_scale (band and
    # planted columns unchanged).
    q_scale: float = 1.0
    # YaRN attention temperature (explainer, "Length Extrapolation"): with
    # s = max(1, seq_len / yarn_train_len), sqrt(1/t) = 0.1 ln(s) + 1 and the logits
    # are divided by t sqrt(D). None: t = 1.
    yarn_train_len: Optional[int] = None
    # planted retrieval columns: K += planted_k u at the planted positions, Q += planted_q u
    planted_q: float = 1.5
    planted_k: float = 4.0
    # scaled logit added inside the aligned 64 x 64 diagonal blocks (the band clause)
    band_logit: float = 2.0

    @property
    def dca_window(self) -> Optional[int]:
        return None if self.dca_chunk is None else self.dca_chunk // 32

    @property
    def dca_stride(self) -> Optional[int]:
        return None if self.dca_chunk is None else self.dca_chunk - self.dca_chunk // 32

    @property
    def yarn_factor(self) -> float:
        """1 / t of the YaRN temperature (1.0 without YaRN)."""
        if self.yarn_train_len is None:
            return 1.0
        s = max(1.0, self.seq_len / self.yarn_train_len)
        return (0.1 * math.log(s) + 1.0) ** 2

    @property
    def softmax_scale(self) -> float:
        """The scale of q.k in the softmax: 1 / (t sqrt(D))."""
        return self.yarn_factor / math.sqrt(self.head_dim)

    @property
    def group(self) -> int:
        return self.hq // self.hkv

    @property
    def n_chunks(self) -> int:
        return (self.seq_len + self.chunk - 1) // self.chunk

    def chunk_bounds(self, c: int) -> tuple[int, int]:
        cs = c * self.chunk
        return cs, min(cs + self.chunk, self.seq_len)


WORKLOADS: dict[int, Workload] = {
    1: Workload("cfg1_h2x1_n4k", hq=2, hkv=1, seq_len=4096, seed=0, n_planted=16,
                kv_budget=256, ks_budget=256, refine_tau=None),
    2: Workload("cfg2_qwen7b_n32k_refine", hq=28, hkv=4, seq_len=32768, seed=1, n_planted=64,
                kv_budget=1000, ks_budget=2048, refine_tau=0.9),
    3: Workload("cfg3_qwen7b_n128k_4chunks_refine", hq=28, hkv=4, seq_len=131072, seed=2,
                n_planted=64, kv_budget=1000, ks_budget=2048, refine_tau=0.9),
    4: Workload("cfg4_14b_n256k_dca64k", hq=40, hkv=8, seq_len=262144, seed=3, n_planted=256,
                kv_budget=1000, ks_budget=2048, refine_tau=None, dca_chunk=65536),
    5: Workload("cfg5_14b_n1m_dca256k_refine", hq=40, hkv=8, seq_len=1048576, seed=4,
                n_planted=1024, kv_budget=1000, ks_budget=2048, refine_tau=0.9,
                dca_chunk=262144),
    # Next rows: the sparse regime (peaked base logits, std 4) of configs 2 and 5, and
    # config 5 with the YaRN temperature for 1M tokens over a 262,144-token training length.
    6: Workload("cfg6_qwen7b_n32k_refine_peaked", hq=28, hkv=4, seq_len=32768, seed=1, n_planted=64,
                kv_budget=1000, ks_budget=2048, refine_tau=0.9, q_scale=4.0),
    7: Workload("cfg7_14b_n1m_dca256k_refine_peaked", hq=40, hkv=8, seq_len=1048576, seed=4,
                n_planted=1024, kv_budget=1000, ks_budget=2048, refine_tau=0.9, dca_chunk=262144,
                q_scale=4.0),
    8: Workload("cfg8_14b_n1m_dca256k_refine_yarn", hq=40, hkv=8, seq_len=1048576, seed=4,
                n_planted=1024, kv_budget=1000, ks_budget=2048, refine_tau=0.9, dca_chunk=262144,
                yarn_train_len=262144),
    # A regime where vertical-slash structure exists: config 5 with the diagonal band at
    # +15 scaled logits, the planted columns at +10.7 (11 x 11 raw) and the queries' N(0, 1)
    # part halved. Refinement stops at the base budgets; the selection is the band's
    # offsets, offset runs that the planted columns induce in the estimation rows, and the
    # planted columns themselves, scattered over the sequence.
    9: Workload("cfg9_14b_n1m_dca256k_refine_structured", hq=40, hkv=8, seq_len=1048576, seed=4,
                n_planted=1024, kv_budget=1000, ks_budget=2048, refine_tau=0.9, dca_chunk=262144,
                q_scale=0.5, band_logit=15.0, planted_q=11.0, planted_k=11.0),
}


def small_workload(base: int, seq_len: int, chunk: int, *, hq: Optional[int] = None,
                   hkv: Optional[int] = None, n_planted: Optional[int] = None,
                   kv_budget: Optional[int] = None, ks_budget: Optional[int] = None,
                   dca_chunk: Optional[int] = None, seed: Optional[int] = None,
                   refine_tau: Optional[float] = -1.0, head_dim: Optional[int] = None,
                   q_scale: Optional[float] = None, yarn_train_len: Optional[int] = None,
                   name: Optional[str] = None, **extra) -> Workload:
    """A reduced copy of workload `base` (same generator recipe, smaller sizes)."""
    w = WORKLOADS[base]
    kw = dict(seq_len=seq_len, chunk=chunk)
    if hq is not None:
        kw["hq"] = hq
    if hkv is not None:
        kw["hkv"] = hkv
    if n_planted is not None:
        kw["n_planted"] = n_planted
    if kv_budget is not None:
        kw["kv_budget"] = kv_budget
    if ks_budget is not None:
        kw["ks_budget"] = ks_budget
    if dca_chunk is not None:
        kw["dca_chunk"] = dca_chunk
    if seed is not None:
        kw["seed"] = seed
    if refine_tau != -1.0:
        kw["refine_tau"] = refine_tau
    if head_dim is not None:
        kw["head_dim"] = head_dim
    if q_scale is not None:
        kw["q_scale"] = q_scale
    if yarn_train_len is not None:
        kw["yarn_train_len"] = yarn_train_len
    kw.update(extra)
    kw["name"] = name or f"{w.name}_small_n{seq_len}_c{chunk}"
    return replace(w, **kw)
