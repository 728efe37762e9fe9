"""CPU oracle for the sparse-prefill path (TEST INFRASTRUCTURE ONLY).

A plain, slow, float64 numpy restatement of what the path computes: RoPE with
the rotate-half convention, Dual Chunk Attention position remapping, last-64
query estimation, vertical/slash top-k selection, attention-recall refinement
and the masked softmax attention, over a chunked prefill. It shares no code with
the CUDA library and imports nothing from it.

Only the tests, `__graft_entry__.smoke()` and the `cpu_baseline` / reference arm
of `bench.py` may import or execute anything in this package; the library's
product path never does.

Parity pins: every function is pinned by tests under `tests/` marked
`not gpu` (pure-Python brute force on tiny inputs, closed forms and invariants);
see `tests/test_oracle_pins.py`. The readings that the pages leave open
(local window W = C/32, the doubling rule, mean-over-rows recall, the forced
slash offset 0) are fixed so that both sides agree but are "parity unpinned"
against the pages themselves.
"""
from .vs_oracle import (
    attention_rows,
    attention_rows_dense,
    bf16_rne,
    dca_positions,
    dca_q_position,
    estimate,
    inv_freq,
    layer_prefill,
    recall,
    refine,
    rope,
    select,
    topk_sorted,
)

__all__ = [
    "attention_rows",
    "attention_rows_dense",
    "bf16_rne",
    "dca_positions",
    "dca_q_position",
    "estimate",
    "inv_freq",
    "layer_prefill",
    "recall",
    "refine",
    "rope",
    "select",
    "topk_sorted",
]
