"""Work counts of the reported metrics, from a workload's shapes and class maps alone.

Pure numpy: this module loads no library and computes no attention, so the benchmark's oracle arm can
count the same visible FLOPs as the GPU arm without mapping libsegpaged.so.

* ``visible_counts`` -- |V(i)| for every query position of one (sequence, KV head): all i + 1 keys of
  the causal context for a global head; for a local head the sink keys j < min(S, i + 1) plus the
  window keys max(i - W + 1, 0) <= j <= i, counted once where the two ranges overlap.
* ``visible_flops`` -- 4 * D * sum |V(i)| over (query row, query head): 2 FLOPs for Q.K and 2 for P.V
  per visible (query, key, dimension), the algorithmic work of prefill (masked or skipped work is not
  counted).
* ``mass_pairs`` -- visible (query row, query head, key inside the query range) triples: one
  exponential each in the token-mass pass.
"""
from __future__ import annotations

import numpy as np


def visible_counts(w, layer: int, b: int, kh: int) -> np.ndarray:
    """|V(i)| for every query position of (sequence b, KV head kh) of a layer."""
    L, Lq = w.ctx_lens[b], w.q_lens[b]
    i = np.arange(L - Lq, L, dtype=np.int64)
    g, S, W = (int(x) for x in w.classes[layer, b, kh])
    if g:
        return i + 1
    sink = np.minimum(S, i + 1)
    lo = np.maximum(i - W + 1, 0)
    return sink + (i + 1 - lo) - np.clip(sink - lo, 0, None)


def visible_flops(w, layers=None) -> float:
    """4 * D * sum over (sequence, query head, query row) of |V(i)|: the algorithmic FLOPs of prefill."""
    total = 0.0
    for li in (range(w.layers) if layers is None else layers):
        for b in range(w.num_seqs):
            for kh in range(w.num_kv_heads):
                total += 4.0 * w.head_dim * w.group * float(visible_counts(w, li, b, kh).sum())
    return total


def mass_pairs(w, layer: int) -> int:
    """Visible (query row, query head, key of the query range) triples of one layer: one exp2 each."""
    total = 0
    for b in range(w.num_seqs):
        L, Lq = w.ctx_lens[b], w.q_lens[b]
        j = np.arange(L - Lq, L, dtype=np.int64)
        for kh in range(w.num_kv_heads):
            g, S, W = (int(x) for x in w.classes[layer, b, kh])
            n = (L - j) if g else np.where(j < S, L - j, np.minimum(L - j, W))
            total += w.group * int(n.sum())
    return total
