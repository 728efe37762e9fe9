"""Seeded generator of pre-RoPE Q, K, V for one attention layer.

Recipe (one torch CPU generator per (seed, tensor, head), so any head can be
regenerated alone; all arithmetic in fp32, one final round-to-nearest-even cast
to bf16):

* Q [Hq, N, D], K and V [Hkv, N, D]: iid N(0, 1).
* Planted vertical columns: `n_planted` distinct uniform positions in [0, N),
  the same for every KV head. u is a random unit vector on the 8 dims of the
  four lowest-frequency rotary pairs (dims 60..63 and 124..127 at D = 128),
  which rotate by under 0.3 rad across 1M positions at base 1e7, so the
  attraction survives RoPE at any distance. K[:, p] += 4 u at planted p and
  Q[:, i] += 1.5 u for every head and position.
* Local band ("q_i . k_j += 2 for i - j < 64", in scaled-logit units): for every
  64-aligned block b a random unit vector z_b on the 32 dims of rotary pairs
  32..47 (which turn by at most ~0.02 rad over 64 positions); with
  a = sqrt(band_logit sqrt(D)), Q[:, i] += a z_{i // 64} and K[:, j] += a z_{j // 64},
  which adds band_logit (2) to the scaled logit of every pair inside an aligned
  64 x 64 diagonal block.
* V carries no structure.
* Sparse-regime variant (q_scale != 1): the N(0, 1) part of Q is multiplied by
  q_scale before the structure is added, so base scaled logits have std q_scale.
* Strengths: the band adds band_logit (default 2) scaled logits; the planted
  columns use amplitudes planted_q (queries, default 1.5) and planted_k (keys,
  default 4).
"""
from __future__ import annotations

import math
from typing import Optional

import torch

from .configs import Workload

_TENSOR_ID = {"q": 1, "k": 2, "v": 3, "struct": 4}


def _gen(seed: int, tensor: str, head: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed) * 1_000_003 + _TENSOR_ID[tensor] * 10_007 + int(head))
    return g


def _pair_dims(d: int, pairs: range) -> list[int]:
    half = d // 2
    return [m for m in pairs] + [m + half for m in pairs]


def planted_positions(w: Workload) -> torch.Tensor:
    g = _gen(w.seed, "struct", 0)
    n = min(w.n_planted, w.seq_len)
    perm = torch.randperm(w.seq_len, generator=g)[:n]
    return torch.sort(perm).values


def structure(w: Workload) -> dict:
    """The shared structure vectors: u [D], z [n_blocks, D], planted positions."""
    d = w.head_dim
    half = d // 2
    g = _gen(w.seed, "struct", 1)
    # u: lowest-frequency four pairs (the last four of each half)
    low = range(half - 4, half)
    u = torch.zeros(d, dtype=torch.float32)
    uv = torch.randn(8, generator=g, dtype=torch.float32)
    u[_pair_dims(d, low)] = uv / uv.norm()
    # z_b: pairs in the upper-middle band (32..47 at D=128), scaled with D
    zpairs = range(half // 2, half // 2 + half // 4)
    zd = _pair_dims(d, zpairs)
    nb = (w.seq_len + 63) // 64
    zr = torch.randn(nb, len(zd), generator=g, dtype=torch.float32)
    zr = zr / zr.norm(dim=1, keepdim=True)
    z = torch.zeros(nb, d, dtype=torch.float32)
    z[:, zd] = zr
    return {"u": u, "z": z, "planted": planted_positions(w)}


def _band_amp(d: int, logit: float = 2.0) -> float:
    return math.sqrt(logit * math.sqrt(d))


def generate_head(w: Workload, tensor: str, head: int, rows: Optional[torch.Tensor] = None,
                  st: Optional[dict] = None) -> torch.Tensor:
    """One head of Q, K or V as bf16 [N, D] (or only `rows`, bit-identical to the
    same rows of the full head)."""
    if st is None:
        st = structure(w)
    n, d = w.seq_len, w.head_dim
    x = torch.randn(n, d, generator=_gen(w.seed, tensor, head), dtype=torch.float32)
    if rows is not None:
        x = x[rows]
        pos = rows
    else:
        pos = torch.arange(n)
    if tensor == "q":
        if w.q_scale != 1.0:
            x *= w.q_scale  # sparse-regime variant: base logits with std q_scale
        x += w.planted_q * st["u"]
        x += _band_amp(d, w.band_logit) * st["z"][pos // 64]
    elif tensor == "k":
        x += _band_amp(d, w.band_logit) * st["z"][pos // 64]
        planted = st["planted"]
        if rows is None:
            x[planted] += w.planted_k * st["u"]
        else:
            hit = torch.isin(pos, planted)
            x[hit] += w.planted_k * st["u"]
    return x.to(torch.bfloat16)


def generate_layer(w: Workload, with_v: bool = True) -> dict:
    """All heads: q [Hq, N, D], k [Hkv, N, D], v [Hkv, N, D] (bf16, CPU)."""
    st = structure(w)
    q = torch.stack([generate_head(w, "q", h, st=st) for h in range(w.hq)])
    k = torch.stack([generate_head(w, "k", h, st=st) for h in range(w.hkv)])
    out = {"q": q, "k": k, "structure": st}
    if with_v:
        out["v"] = torch.stack([generate_head(w, "v", h, st=st) for h in range(w.hkv)])
    return out
