"""Seeded synthetic workloads for SegPagedAttention prefill.

Shapes, head-class maps, input tensors and physical page assignments of the five layer workloads
the library is measured on. This module holds none of the method's arithmetic: it never decides
which pages a head stores (page counts come in as arguments) and computes no attention. Both the
CUDA path and the CPU oracle take their inputs from here.

Recipe (all bf16 values are float32 draws rounded to bf16):
  * Q, K, V ~ N(0, 1), drawn with torch's generator seeded per (workload, layer, tensor).
  * ``low_rank_bias``: K and Q get 2 * A @ B_k^T added before rounding, with B_k an orthonormal
    D x 4 basis per KV head and A ~ N(0, 1) (own draw for K and for Q), so scores concentrate.
  * Class maps: a global KV head index drawn per sequence (or per layer) from the workload seed.
  * Page order: "shuffled" = a seeded permutation of all physical ids; "interleaved" = ids handed
    out round-robin over sequences (and heads) in logical-page order.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch


@dataclass
class Workload:
    name: str
    ctx_lens: list            # L_b
    q_lens: list              # Lq_b (tail query rows)
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    page_size: int
    classes: np.ndarray       # [layers, B, Hkv, 3] int32 (is_global, sink, window)
    seed: int
    page_order: str = "shuffled"
    low_rank_bias: bool = False
    rope_theta: float | None = None
    rope_deltas: list | None = None
    description: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def layers(self) -> int:
        return self.classes.shape[0]

    @property
    def num_seqs(self) -> int:
        return len(self.ctx_lens)

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def total_q(self) -> int:
        return int(sum(self.q_lens))

    @property
    def total_k(self) -> int:
        return int(sum(self.ctx_lens))

    def cu_q(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.q_lens)]).astype(np.int32)

    def cu_k(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.ctx_lens)]).astype(np.int32)


def _local(S, W):
    return (0, S, W)


GLOBAL = (1, 0, 0)


def tiny() -> Workload:
    """1 sequence, L=256, Lq=64, 4 query / 2 KV heads, D=64, P=16; KV head 0 global, 1 local (S=4, W=64)."""
    cls = np.array([[[GLOBAL, _local(4, 64)]]], dtype=np.int32)
    return Workload("tiny", [256], [64], 4, 2, 64, 16, cls, seed=1001, page_order="shuffled",
                    description="tiny SegPaged prefill layer: L=256, Lq=64, Hq=4, Hkv=2, D=64, P=16")


def mistral_7b() -> Workload:
    """Mistral-7B-shaped layer: L=8192, Lq=512, 32/8 heads, D=128, P=64, 1 global KV head, 7 local
    (S=64, W=1024); the build re-rotates keys by a RoPE delta (theta 1e6, delta ~ U[0, 4096))."""
    rng = np.random.default_rng(1002)
    g = int(rng.integers(8))
    row = [GLOBAL if k == g else _local(64, 1024) for k in range(8)]
    delta = [int(rng.integers(0, 4096))]
    return Workload("mistral-7b", [8192], [512], 32, 8, 128, 64, np.array([[row]], np.int32), seed=1002,
                    rope_theta=1e6, rope_deltas=delta,
                    description="Mistral-7B-shaped layer: L=8192, Lq=512, Hq=32, Hkv=8, D=128, P=64")


def llama_70b(globals_per_seq: int = 1) -> Workload:
    """Llama-3.3-70B-shaped batched layer: 4 sequences, L_b ~ U[16384, 32768], Lq=2048 each, 64/8 heads,
    D=128, P=64; per sequence `globals_per_seq` global KV heads, the rest local (S=128, W=2048);
    physical pages interleaved across sequences."""
    rng = np.random.default_rng(1003)
    L = [int(x) for x in rng.integers(16384, 32769, size=4)]
    rows = []
    for _ in range(4):
        gs = set(int(x) for x in rng.choice(8, size=globals_per_seq, replace=False))
        rows.append([GLOBAL if k in gs else _local(128, 2048) for k in range(8)])
    return Workload(f"llama-3.3-70b" + ("" if globals_per_seq == 1 else f"-g{globals_per_seq}"), L, [2048] * 4,
                    64, 8, 128, 64, np.array([rows], np.int32), seed=1003, page_order="interleaved",
                    description="Llama-3.3-70B-shaped layer: 4 seqs, L~U[16K,32K], Lq=2048, Hq=64, Hkv=8, D=128, P=64")


def qwen3_32b(globals_: int = 1) -> Workload:
    """Qwen3-32B-shaped long context: L=131072, chunked prefill of Lq=8192 tail queries, 64/8 heads, D=128,
    P=128, low-rank-biased K and Q; `globals_` global KV heads, the rest local (S=128, W=4096)."""
    rng = np.random.default_rng(1004)
    gs = set(int(x) for x in rng.choice(8, size=globals_, replace=False))
    row = [GLOBAL if k in gs else _local(128, 4096) for k in range(8)]
    return Workload("qwen3-32b" + ("" if globals_ == 1 else f"-g{globals_}"), [131072], [8192], 64, 8, 128, 128,
                    np.array([[row]], np.int32), seed=1004, low_rank_bias=True,
                    description="Qwen3-32B-shaped layer: L=131072, Lq=8192, Hq=64, Hkv=8, D=128, P=128")


def qwen3_32b_small_q(lq: int) -> Workload:
    """Decode-like probe on the Qwen3-32B-shaped layer: the same L=131072 pool and class map, only the last
    `lq` positions queried (Lq in {16, 64}), so the KV pages dominate the bytes moved."""
    w = qwen3_32b()
    w.name = f"qwen3-32b-lq{lq}"
    w.q_lens = [lq]
    w.description = f"Qwen3-32B-shaped decode-like probe: L=131072, Lq={lq}, Hq=64, Hkv=8, D=128, P=128"
    return w


def llama_70b_decode(num_seqs: int = 32, lq: int = 16) -> Workload:
    """Decode-like batch on Llama-3.3-70B-shaped heads: `num_seqs` sequences with L_b ~ U[16384, 32768], each
    querying only its last `lq` positions (a multi-token decode or draft-verification step), 64/8 heads, D=128,
    P=64; per sequence one global KV head at a seeded index, the rest local (S=128, W=2048); pages interleaved
    across sequences. The stored pages dominate the bytes moved, so the launch is HBM-bound."""
    rng = np.random.default_rng(1006)
    L = [int(x) for x in rng.integers(16384, 32769, size=num_seqs)]
    rows = []
    for _ in range(num_seqs):
        g = int(rng.integers(8))
        rows.append([GLOBAL if k == g else _local(128, 2048) for k in range(8)])
    return Workload(f"llama-3.3-70b-decode{num_seqs}x{lq}", L, [lq] * num_seqs, 64, 8, 128, 64,
                    np.array([rows], np.int32), seed=1006, page_order="interleaved",
                    description=f"Llama-3.3-70B-shaped decode-like batch: {num_seqs} seqs, L~U[16K,32K], Lq={lq}, "
                                f"Hq=64, Hkv=8, D=128, P=64")


def dsv4_flash(layers: int = 43) -> Workload:
    """DeepSeek-V4-Flash-style head split: `layers` layers of 64 MHA heads (own KV each), D=128, one sequence
    L=131072 with Lq=4096, P=128, fully shuffled pool. Layers 0-2 and the last three are all global;
    the others have 8 global heads (seeded per layer) and 56 local heads (S=128, W=4096)."""
    rng = np.random.default_rng(1005)
    cls = np.zeros((layers, 1, 64, 3), np.int32)
    for layer in range(layers):
        if layer < 3 or layer >= layers - 3:
            cls[layer, 0, :] = GLOBAL
        else:
            gs = set(int(x) for x in rng.choice(64, size=8, replace=False))
            for k in range(64):
                cls[layer, 0, k] = GLOBAL if k in gs else _local(128, 4096)
    return Workload("dsv4-flash", [131072], [4096], 64, 64, 128, 128, cls, seed=1005,
                    description=f"DeepSeek-V4-Flash-style: {layers} layers, 64 MHA heads, L=131072, Lq=4096, D=128, P=128")


def custom(name: str, seqs, num_q_heads: int, num_kv_heads: int, head_dim: int, page_size: int, classes, seed: int,
           page_order: str = "shuffled", rope_theta=None, rope_deltas=None, low_rank_bias=False) -> Workload:
    """Any single-layer shape: seqs = [(L, Lq)], classes = [B][Hkv] of (is_global, sink, window)."""
    cls = np.asarray(classes, np.int32)[None]
    return Workload(name, [s[0] for s in seqs], [s[1] for s in seqs], num_q_heads, num_kv_heads, head_dim, page_size,
                    cls, seed=seed, page_order=page_order, low_rank_bias=low_rank_bias, rope_theta=rope_theta,
                    rope_deltas=rope_deltas, description=name)


WORKLOADS = {
    "tiny": tiny,
    "mistral-7b": mistral_7b,
    "llama-3.3-70b": llama_70b,
    "qwen3-32b": qwen3_32b,
    "dsv4-flash": dsv4_flash,
    "qwen3-32b-lq16": lambda: qwen3_32b_small_q(16),
    "qwen3-32b-lq64": lambda: qwen3_32b_small_q(64),
    "llama-3.3-70b-decode32x16": lambda: llama_70b_decode(32, 16),
}


def get(name: str) -> Workload:
    return WORKLOADS[name]()


# --------------------------------------------------------------------------------------- tensors

def _orthonormal(gen: torch.Generator, D: int, r: int) -> torch.Tensor:
    a = torch.randn(D, r, generator=gen, dtype=torch.float32, device=gen.device)
    qm, _ = torch.linalg.qr(a.cpu())
    return qm.to(gen.device)


def layer_inputs(w: Workload, layer: int = 0, device="cpu", parts: str = "qkv"):
    """(q [total_q, Hq, D], k [total_k, Hkv, D], v [total_k, Hkv, D]) bf16 tensors of one layer.

    Draws happen on `device` with a generator seeded from (workload seed, layer), so a given device
    type always produces the same values. The three tensors use separate generator streams, so
    parts="q" returns the same Q (and None for K, V) without drawing K and V.
    """
    dev = torch.device(device)
    base = w.seed * 1000 + layer * 10

    def gen(i):
        g = torch.Generator(device=dev)
        g.manual_seed(base + i)
        return g

    D = w.head_dim
    want_kv = parts == "qkv"
    q = torch.randn(w.total_q, w.num_q_heads, D, generator=gen(0), device=dev, dtype=torch.float32)
    k = v = None
    if want_kv:
        k = torch.randn(w.total_k, w.num_kv_heads, D, generator=gen(1), device=dev, dtype=torch.float32)
        v = torch.randn(w.total_k, w.num_kv_heads, D, generator=gen(2), device=dev, dtype=torch.float32)
    if w.low_rank_bias:
        gb = gen(3)
        basis = torch.stack([_orthonormal(gb, D, 4) for _ in range(w.num_kv_heads)])        # [Hkv, D, 4]
        ak = torch.randn(w.total_k, w.num_kv_heads, 4, generator=gb, device=dev)
        if want_kv:
            k += 2.0 * torch.einsum("lhr,hdr->lhd", ak, basis)
        aq = torch.randn(w.total_q, w.num_q_heads, 4, generator=gb, device=dev)
        qb = basis.repeat_interleave(w.group, dim=0)                                          # [Hq, D, 4]
        q += 2.0 * torch.einsum("lhr,hdr->lhd", aq, qb)
    bf = torch.bfloat16
    return q.to(bf), (k.to(bf) if want_kv else None), (v.to(bf) if want_kv else None)


# --------------------------------------------------------------------------------- page tables

def assign_pages(counts: np.ndarray, order: str, seed: int, base: int = 0, pool_pages: int | None = None):
    """Physical page ids for per-(sequence, KV head) page counts.

    counts: int [B, Hkv], the stored page count of each head (from the storage accounting).
    Returns (page_table int32 [sum counts], offs int32 [B*Hkv + 1], num_pages). Ids are taken from
    [base, base + sum counts) -- or from a seeded choice out of [0, pool_pages) when pool_pages is given --
    shuffled by the seed, or interleaved round-robin over sequences in logical-page order.
    """
    counts = np.asarray(counts, dtype=np.int64)
    B, H = counts.shape
    flat = counts.reshape(-1)
    offs = np.concatenate([[0], np.cumsum(flat)]).astype(np.int64)
    total = int(offs[-1])
    rng = np.random.default_rng(seed)
    table = np.empty(total, dtype=np.int64)
    if pool_pages is not None:
        ids = rng.choice(pool_pages, size=total, replace=False)
    elif order == "interleaved":
        ids = None
    else:
        ids = base + rng.permutation(total)
    if ids is not None:
        table[:] = ids
    else:
        nxt = base
        for t in range(int(flat.max()) if total else 0):
            for b in range(B):
                for h in range(H):
                    if t < counts[b, h]:
                        table[offs[b * H + h] + t] = nxt
                        nxt += 1
    num_pages = pool_pages if pool_pages is not None else base + total
    return table.astype(np.int32), offs.astype(np.int32), int(num_pages)
