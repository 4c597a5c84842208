"""Shared helpers of the GPU parity tests: oracle inputs and per-KV-head sub-problems.

Tolerances (the method's stated bar for this bf16 path): O max-abs 1e-2 (bf16 output, fp32
accumulation, bf16 probabilities); LSE max-abs 1e-3 (fp32 sums, natural log). Build and gather are
bit-exact.
"""
import math

import numpy as np
import torch

from head_sparse_paged_b200 import synth
from oracle import reference as orc

O_TOL = 1e-2
LSE_TOL = 1e-3


def oracle_dense(w: synth.Workload, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor):
    """float32 numpy copies of the layer inputs as the oracle sees them: keys re-rotated by the
    workload's RoPE delta with the oracle's own table and rounding rule."""
    qn = q.float().cpu().numpy()
    kn = k.float().cpu().numpy()
    vn = v.float().cpu().numpy()
    if w.rope_theta is not None:
        tab = orc.rope_cos_sin(w.rope_theta, w.rope_deltas, w.head_dim)
        cu = w.cu_k()
        for b in range(w.num_seqs):
            kn[cu[b]:cu[b + 1]] = orc.rope_rotate_bf16(kn[cu[b]:cu[b + 1]], tab[b])
    return qn, kn, vn


def full_problem(w: synth.Workload, layer: int, qn, kn, vn) -> orc.Problem:
    c = w.classes[layer]
    return orc.Problem(qn, kn, vn, w.cu_q(), w.cu_k(), c[..., 0], c[..., 1], c[..., 2])


def head_problem(w: synth.Workload, layer: int, b: int, kh: int, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor):
    """Sub-problem of one (sequence, KV head): its query rows and G query heads, its keys and values."""
    G = w.group
    cq, ck = w.cu_q(), w.cu_k()
    qs = q[cq[b]:cq[b + 1], kh * G:(kh + 1) * G].float().cpu().numpy()
    ks = k[ck[b]:ck[b + 1], kh:kh + 1].float().cpu().numpy()
    vs = v[ck[b]:ck[b + 1], kh:kh + 1].float().cpu().numpy()
    if w.rope_theta is not None:
        ks = orc.rope_rotate_bf16(ks, orc.rope_cos_sin(w.rope_theta, [w.rope_deltas[b]], w.head_dim)[0])
    g, S, W = (int(x) for x in w.classes[layer, b, kh])
    L, Lq = w.ctx_lens[b], w.q_lens[b]
    return orc.Problem(qs, ks, vs, np.array([0, Lq], np.int32), np.array([0, L], np.int32),
                       np.array([[g]]), np.array([[S]]), np.array([[W]]))


def sample_rows(Lq: int, npos: int, rng, extra: int = 5):
    rows = {0, 1, npos - 1, npos, Lq // 2, Lq - 2, Lq - 1}
    rows |= set(int(x) for x in rng.integers(0, Lq, size=extra))
    return sorted(r for r in rows if 0 <= r < Lq)


def compare(o_gpu: np.ndarray, lse_gpu: np.ndarray, o_ref: np.ndarray, lse_ref: np.ndarray, what=""):
    eo = float(np.max(np.abs(o_gpu.astype(np.float64) - o_ref))) if o_ref.size else 0.0
    el = float(np.max(np.abs(lse_gpu.astype(np.float64) - lse_ref))) if lse_ref.size else 0.0
    assert np.all(np.isfinite(o_gpu)) and np.all(np.isfinite(lse_gpu)), what
    assert eo <= O_TOL and el <= LSE_TOL, f"{what}: max|dO|={eo:.3e} max|dLSE|={el:.3e}"
    return eo, el
