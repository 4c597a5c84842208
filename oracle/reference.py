"""Oracle for SegPagedAttention prefill and build -- TEST INFRASTRUCTURE, not product code.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import this module. The product path (``head_sparse_paged_b200``)
never imports it, and it imports nothing from the product.

Everything here is written from the method's definition, in fp64 where it is floating point:

* ``visible_keys`` -- the sink-plus-window visible set of one query, built from two index
  ranges. Global heads see the whole causal context; local heads keep only their sink tokens
  and their recent window ("RedKnot" write-up, bjdmk.com.cn, section 二 "三大核心机制", item 3
  "SegPagedAttention"; shshi.cn, "RedKnot技术原理" 1). The pages give no boundaries; the reading
  used here: key j is visible to query i iff j <= i and (head is global, or j < S, or j > i - W).
* ``attention`` -- exact softmax attention over that set (naive two-pass softmax), plus the
  natural-log LSE.
* ``stored_logical_pages`` -- which logical pages of a (sequence, KV head) a SegPaged pool keeps:
  all of them for a global head; the sink pages and the pages any served query's window can
  reach for a local head ("局部头物理上只存 sink + 最近窗口的 KV 页", bjdmk.com.cn, section 二 item 3).
* ``build_pool`` -- the pool a build must produce: a bitwise copy of each stored page's rows of
  the dense K/V (zero past the context end), K optionally re-rotated by a RoPE delta
  ("RoPE位置对齐", shshi.cn, "RedKnot技术原理" 2 "位置无关缓存复用").
* ``rope_cos_sin`` / ``rope_rotate_bf16`` -- the RoPE delta rotation, rotate-half pairing
  (d, d + D/2), with the bit-exact fp32 rule stated in their docstrings.
* ``rope_fragment_of`` / ``rope_fragment_keys`` -- the same re-alignment applied per fragment of a
  sequence (reused document fragments sitting at other offsets than the ones their keys were
  computed at: shshi.cn, "RedKnot技术原理" 2 "位置无关缓存复用"). Reading: a token belongs to the
  last fragment that starts at or before it; tokens before the first fragment keep their keys.
* ``token_mass`` / ``select_topk`` -- the token score of the sparse-FFN selection (top-k tokens by
  attention score run the dense FFN, the rest take the residual path: shshi.cn, "RedKnot技术原理" 3
  "稀疏FFN动态调度"). The pages define neither the score nor ties; the reading used here: a token's
  score is the attention mass it receives from every query row and head of the prefill, and among
  equal scores the lower row is chosen.

``OracleLib`` wraps the C oracle (segpaged_oracle.c), which forms the visible set by brute-force
predicate scan instead of ranges; the tests require both to agree.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "liboracle.so")


# ----------------------------------------------------------------------------------------------
# Visibility and attention (definition)
# ----------------------------------------------------------------------------------------------

def visible_keys(is_global: bool, sink: int, window: int, i: int) -> np.ndarray:
    """Sorted key positions j visible to the query at absolute position i.

    Global head: [0, i]. Local head: [0, min(S, i+1)) united with [max(i-W+1, 0), i].
    """
    if is_global:
        return np.arange(0, i + 1, dtype=np.int64)
    sink_part = np.arange(0, min(sink, i + 1), dtype=np.int64)
    win_part = np.arange(max(i - window + 1, 0), i + 1, dtype=np.int64)
    return np.union1d(sink_part, win_part)


@dataclass
class Problem:
    """A varlen prefill problem in the layout the library uses.

    q: [total_q, Hq, D]; k, v: [total_k, Hkv, D] (dense, unpaged); cu_q, cu_k: [B+1];
    is_global, sink, window: [B, Hkv]. Values are float arrays holding bf16-representable
    numbers. Query row r of sequence b sits at position L_b - Lq_b + (r - cu_q[b]).
    """
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    cu_q: np.ndarray
    cu_k: np.ndarray
    is_global: np.ndarray
    sink: np.ndarray
    window: np.ndarray

    @property
    def B(self):
        return len(self.cu_q) - 1

    @property
    def Hq(self):
        return self.q.shape[1]

    @property
    def Hkv(self):
        return self.k.shape[1]

    @property
    def D(self):
        return self.q.shape[2]

    def row_seq_pos(self, r: int):
        b = int(np.searchsorted(self.cu_q, r, side="right") - 1)
        L = int(self.cu_k[b + 1] - self.cu_k[b])
        Lq = int(self.cu_q[b + 1] - self.cu_q[b])
        return b, L - Lq + (r - int(self.cu_q[b]))


def attention_row(pb: Problem, r: int, h: int, scale: float, shift: float = 0.0):
    """O (fp64 [D]), LSE (natural log), probabilities over V(i) and V(i) for query row r, head h.

    ``shift`` is a test hook: a constant added to every visible logit of the row.
    """
    b, i = pb.row_seq_pos(r)
    G = pb.Hq // pb.Hkv
    kh = h // G
    vis = visible_keys(bool(pb.is_global[b, kh]), int(pb.sink[b, kh]), int(pb.window[b, kh]), i)
    rows = int(pb.cu_k[b]) + vis
    kk = pb.k[rows, kh, :].astype(np.float64)
    vv = pb.v[rows, kh, :].astype(np.float64)
    s = scale * (kk @ pb.q[r, h, :].astype(np.float64)) + shift
    m = s.max()
    e = np.exp(s - m)
    lse = m + math.log(e.sum())
    p = np.exp(s - lse)
    return p @ vv, lse, p, vis


def attention(pb: Problem, scale: float, rows=None):
    """O [n, D] and LSE [n] (fp64) for the (row, head) items in ``rows`` (all if None)."""
    if rows is None:
        rows = [(r, h) for r in range(pb.q.shape[0]) for h in range(pb.Hq)]
    o = np.zeros((len(rows), pb.D))
    lse = np.zeros(len(rows))
    for t, (r, h) in enumerate(rows):
        o[t], lse[t], _, _ = attention_row(pb, r, h, scale)
    return o, lse


def token_mass(pb: Problem, scale: float) -> np.ndarray:
    """Attention mass received by each query row's own token, fp64 [total_q].

    mass[r] = sum over query heads h and query rows r' (position i) of p_h(i, j) for j in V_h(i),
    j the position of row r, p the softmax probabilities of ``attention_row``.
    """
    mass = np.zeros(pb.q.shape[0])
    for rr in range(pb.q.shape[0]):
        b, _ = pb.row_seq_pos(rr)
        L = int(pb.cu_k[b + 1] - pb.cu_k[b])
        q0 = L - int(pb.cu_q[b + 1] - pb.cu_q[b])
        for h in range(pb.Hq):
            _, _, p, vis = attention_row(pb, rr, h, scale)
            keep = vis >= q0
            np.add.at(mass, int(pb.cu_q[b]) + (vis[keep] - q0), p[keep])
    return mass


def select_topk(mass: np.ndarray, cu_q, k_per_seq) -> np.ndarray:
    """Global rows chosen per sequence, concatenated in sequence order, each list ascending.

    Sequence b keeps min(max(k_b, 0), Lq_b) rows of largest mass; equal masses prefer the lower row.
    """
    out = []
    for b in range(len(cu_q) - 1):
        lo, hi = int(cu_q[b]), int(cu_q[b + 1])
        kb = min(max(int(k_per_seq[b]), 0), hi - lo)
        rows = sorted(range(lo, hi), key=lambda r: (-mass[r], r))[:kb]
        out.extend(sorted(rows))
    return np.asarray(out, dtype=np.int64)


# ----------------------------------------------------------------------------------------------
# Storage rule, footprint and build
# ----------------------------------------------------------------------------------------------

def stored_logical_pages(L: int, Lq: int, is_global: bool, sink: int, window: int, P: int) -> list[int]:
    """Logical pages (ascending) that a (sequence, KV head) keeps in the pool.

    Global: every page of [0, L). Local: pages holding a sink token [0, min(S, L)) plus pages
    holding a token any served query (positions L-Lq .. L-1) can see in its window, i.e. tokens
    [max(L-Lq-W+1, 0), L).
    """
    n_all = -(-L // P)
    if is_global:
        return list(range(n_all))
    sink_pages = set(range(-(-min(sink, L) // P)))
    lo = max(L - Lq - window + 1, 0)
    win_pages = set(range(lo // P, n_all))
    return sorted(sink_pages | win_pages)


def pages_bytes(cu_k, cu_q, is_global, sink, window, P: int, D: int, elem_bytes: int = 2):
    """(stored K+V bytes, dense K+V bytes, stored page count per (b, k)).

    Dense = every KV head of every sequence keeping all ceil(L/P) pages.
    """
    B, Hkv = is_global.shape
    per = np.zeros((B, Hkv), dtype=np.int64)
    dense_pages = 0
    for b in range(B):
        L = int(cu_k[b + 1] - cu_k[b])
        Lq = int(cu_q[b + 1] - cu_q[b])
        for kh in range(Hkv):
            per[b, kh] = len(stored_logical_pages(L, Lq, bool(is_global[b, kh]), int(sink[b, kh]), int(window[b, kh]), P))
            dense_pages += -(-L // P)
    unit = P * D * 2 * elem_bytes
    return int(per.sum()) * unit, dense_pages * unit, per


def rope_cos_sin(theta: float, deltas, D: int) -> np.ndarray:
    """[B, D/2, 2] float32 table of (cos, sin) of delta_b * theta^(-2d/D), computed in fp64."""
    d = np.arange(D // 2, dtype=np.float64)
    inv_freq = theta ** (-2.0 * d / D)
    ang = np.asarray(deltas, dtype=np.float64)[:, None] * inv_freq[None, :]
    return np.stack([np.cos(ang), np.sin(ang)], axis=-1).astype(np.float32)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32 holding bf16 values."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return (u.astype(np.uint32) << 16).view(np.float32)


def rope_rotate_bf16(x: np.ndarray, cs: np.ndarray) -> np.ndarray:
    """Rotate-half RoPE of keys x [..., D] (bf16 values) by a (cos, sin) table cs [D/2, 2].

    Rule: y1 = x1*c - x2*s and y2 = x2*c + x1*s, each product and each sum rounded to fp32
    (no fused multiply-add), then rounded to bf16 with ties to even.
    """
    D = x.shape[-1]
    x = x.astype(np.float32)
    x1, x2 = x[..., : D // 2], x[..., D // 2:]
    c, s = cs[:, 0], cs[:, 1]
    with np.errstate(over="ignore", invalid="ignore"):
        y1 = np.float32(x1 * c) - np.float32(x2 * s)
        y2 = np.float32(x2 * c) + np.float32(x1 * s)
    return bf16_round(np.concatenate([y1, y2], axis=-1).astype(np.float32))


def rope_fragment_of(starts, tok: int) -> int:
    """Index of the last fragment starting at or before token ``tok`` (starts ascending), or -1."""
    f = -1
    for i, s0 in enumerate(starts):
        if s0 <= tok:
            f = i
    return f


def rope_fragment_keys(k: np.ndarray, cu_k, frag_offs, frag_start, frag_cs) -> np.ndarray:
    """Dense keys [total_k, Hkv, D] (bf16 values) after per-fragment re-alignment: token j of sequence b
    is rotated with the (cos, sin) table frag_cs[f] [D/2, 2] of its fragment f, every KV head alike, by
    ``rope_rotate_bf16``; tokens before the sequence's first fragment are unchanged."""
    out = np.array(k, dtype=np.float32, copy=True)
    for b in range(len(cu_k) - 1):
        lo, hi = int(frag_offs[b]), int(frag_offs[b + 1])
        starts = [int(x) for x in frag_start[lo:hi]]
        for j in range(int(cu_k[b + 1] - cu_k[b])):
            f = rope_fragment_of(starts, j)
            if f >= 0:
                row = int(cu_k[b]) + j
                out[row] = rope_rotate_bf16(k[row], frag_cs[lo + f])
    return out


def rope_rotate_f64(x: np.ndarray, angle_per_dim: np.ndarray) -> np.ndarray:
    """Exact (fp64) rotate-half rotation of x [..., D] by angles [D/2]."""
    D = x.shape[-1]
    x1, x2 = x[..., : D // 2], x[..., D // 2:]
    c, s = np.cos(angle_per_dim), np.sin(angle_per_dim)
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def build_pool(k, v, cu_k, cu_q, is_global, sink, window, P, page_table, page_offs, num_pages, rope_cs=None):
    """Expected (k_pool, v_pool) [num_pages, P, D] after a build.

    Stored page number t of (b, kh) goes to physical page page_table[page_offs[b*Hkv+kh] + t].
    Rows past the sequence end are zero. Pages not referenced by any table are left as NaN
    so a test can tell "untouched" from "written".
    """
    B, Hkv = is_global.shape
    D = k.shape[2]
    kp = np.full((num_pages, P, D), np.nan, dtype=np.float32)
    vp = np.full((num_pages, P, D), np.nan, dtype=np.float32)
    for b in range(B):
        L = int(cu_k[b + 1] - cu_k[b])
        Lq = int(cu_q[b + 1] - cu_q[b])
        for kh in range(Hkv):
            lps = stored_logical_pages(L, Lq, bool(is_global[b, kh]), int(sink[b, kh]), int(window[b, kh]), P)
            base = int(page_offs[b * Hkv + kh])
            for t, lp in enumerate(lps):
                pid = int(page_table[base + t])
                kp[pid] = 0.0
                vp[pid] = 0.0
                lo, hi = lp * P, min(lp * P + P, L)
                if hi > lo:
                    krows = k[int(cu_k[b]) + lo: int(cu_k[b]) + hi, kh, :]
                    if rope_cs is not None:
                        krows = rope_rotate_bf16(krows, rope_cs[b])
                    kp[pid, : hi - lo] = krows
                    vp[pid, : hi - lo] = v[int(cu_k[b]) + lo: int(cu_k[b]) + hi, kh, :]
    return kp, vp


# ----------------------------------------------------------------------------------------------
# C oracle (brute-force visible set, OpenMP over rows)
# ----------------------------------------------------------------------------------------------

class OracleLib:
    """ctypes wrapper of liboracle.so (built by oracle/build.py)."""

    def __init__(self, path: str = LIB_PATH):
        if not os.path.exists(path):
            from oracle.build import build_oracle
            build_oracle()
        self.lib = ctypes.CDLL(path)
        p = ctypes.c_void_p
        self.lib.oracle_attention.restype = ctypes.c_int
        self.lib.oracle_attention.argtypes = [ctypes.c_int] * 4 + [p] * 8 + [p, ctypes.c_int64, ctypes.c_double, p, p, p]
        self.lib.oracle_probs.restype = ctypes.c_int64
        self.lib.oracle_probs.argtypes = [ctypes.c_int] * 4 + [p] * 7 + [ctypes.c_int64, ctypes.c_int64, ctypes.c_double, p]
        self.lib.oracle_token_mass.restype = ctypes.c_int
        self.lib.oracle_token_mass.argtypes = [ctypes.c_int] * 4 + [p] * 7 + [ctypes.c_double, p]

    @staticmethod
    def _ptr(a):
        return a.ctypes.data_as(ctypes.c_void_p)

    def _common(self, pb: Problem):
        keep = dict(
            cu_q=np.ascontiguousarray(pb.cu_q, dtype=np.int32),
            cu_k=np.ascontiguousarray(pb.cu_k, dtype=np.int32),
            g=np.ascontiguousarray(pb.is_global.reshape(-1), dtype=np.int32),
            s=np.ascontiguousarray(pb.sink.reshape(-1), dtype=np.int32),
            w=np.ascontiguousarray(pb.window.reshape(-1), dtype=np.int32),
            q=np.ascontiguousarray(pb.q, dtype=np.float32),
            k=np.ascontiguousarray(pb.k, dtype=np.float32),
            v=np.ascontiguousarray(pb.v, dtype=np.float32),
        )
        return keep

    def attention(self, pb: Problem, scale: float, items=None, shift=None):
        """O [n, D] and LSE [n] (fp64). items: int array [n, 2] of (global query row, query head)."""
        a = self._common(pb)
        if items is None:
            items = np.array([(r, h) for r in range(pb.q.shape[0]) for h in range(pb.Hq)], dtype=np.int64)
        items = np.ascontiguousarray(np.asarray(items, dtype=np.int64).reshape(-1, 2))
        n = items.shape[0]
        o = np.zeros((n, pb.D), dtype=np.float64)
        lse = np.zeros(n, dtype=np.float64)
        sh = None if shift is None else np.ascontiguousarray(np.broadcast_to(np.asarray(shift, np.float64), (n,)))
        rc = self.lib.oracle_attention(pb.B, pb.Hq, pb.Hkv, pb.D, self._ptr(a["cu_q"]), self._ptr(a["cu_k"]),
                                       self._ptr(a["g"]), self._ptr(a["s"]), self._ptr(a["w"]),
                                       self._ptr(a["q"]), self._ptr(a["k"]), self._ptr(a["v"]),
                                       self._ptr(items), n, float(scale),
                                       None if sh is None else self._ptr(sh), self._ptr(o), self._ptr(lse))
        if rc != 0:
            raise ValueError("oracle_attention: malformed item")
        return o, lse

    def probs(self, pb: Problem, r: int, h: int, scale: float):
        """Probability row over all keys of the row's sequence, and |V(i)|."""
        a = self._common(pb)
        b, _ = pb.row_seq_pos(r)
        L = int(pb.cu_k[b + 1] - pb.cu_k[b])
        p = np.zeros(max(L, 1), dtype=np.float64)
        n = self.lib.oracle_probs(pb.B, pb.Hq, pb.Hkv, pb.D, self._ptr(a["cu_q"]), self._ptr(a["cu_k"]),
                                  self._ptr(a["g"]), self._ptr(a["s"]), self._ptr(a["w"]),
                                  self._ptr(a["q"]), self._ptr(a["k"]), int(r), int(h), float(scale), self._ptr(p))
        if n < 0:
            raise ValueError("oracle_probs: malformed item")
        return p[:L], int(n)

    def token_mass(self, pb: Problem, scale: float) -> np.ndarray:
        """Attention mass received by each query row's token, fp64 [total_q] (brute-force visible set)."""
        a = self._common(pb)
        m = np.zeros(max(pb.q.shape[0], 1), dtype=np.float64)
        rc = self.lib.oracle_token_mass(pb.B, pb.Hq, pb.Hkv, pb.D, self._ptr(a["cu_q"]), self._ptr(a["cu_k"]),
                                        self._ptr(a["g"]), self._ptr(a["s"]), self._ptr(a["w"]),
                                        self._ptr(a["q"]), self._ptr(a["k"]), float(scale), self._ptr(m))
        if rc != 0:
            raise ValueError("oracle_token_mass failed")
        return m[: pb.q.shape[0]]
