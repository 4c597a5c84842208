"""Host-side checks of the C ABI (no GPU): exported symbols, storage accounting, planner, RoPE table and
argument validation. Expected values come from the oracle (oracle/reference.py)."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

from head_sparse_paged_b200 import segpaged as sp
from head_sparse_paged_b200 import synth
from oracle import reference as orc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# Plan record field positions (head_sparse_paged_b200/csrc/plan.h).
(U_QROW, U_POS0, U_NPOS, U_KVH, U_TOFF, U_NSINK, U_W0, U_GLOBAL, U_SINK, U_WIN, U_AN, U_B0, U_BN, U_NTILES, U_TOTAL,
 U_SEQ, U_T0, U_PART, U_HALF, U_NSPLIT) = range(20)


def test_library_exports_every_declared_symbol():
    hdr = open(os.path.join(ROOT, "include", "segpaged.h")).read()
    declared = set(re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\*?\s+\*?(segpaged_[a-z_]+)\s*\(", hdr, re.M))
    assert declared == set(sp.EXPORTS), declared
    lib = ctypes.CDLL(sp.LIB_PATH)
    for name in declared:
        assert hasattr(lib, name), name


def _all_layer_cases():
    out = []
    for name in ("tiny", "mistral-7b", "llama-3.3-70b", "qwen3-32b"):
        w = synth.get(name)
        out.append((name, w, 0))
    w = synth.dsv4_flash()
    out += [("dsv4-flash-l0", w, 0), ("dsv4-flash-l3", w, 3)]
    return out


@pytest.mark.parametrize("case", range(6))
def test_pages_bytes_matches_oracle(case):
    name, w, layer = _all_layer_cases()[case]
    dims = sp.Dims(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, w.page_size)
    cls = w.classes[layer]
    stored, dense, per = sp.segpaged_pages_bytes(dims, w.ctx_lens, w.q_lens, cls)
    o_stored, o_dense, o_per = orc.pages_bytes(w.cu_k(), w.cu_q(), cls[..., 0], cls[..., 1], cls[..., 2], w.page_size, w.head_dim)
    assert stored == o_stored and dense == o_dense
    assert per.tolist() == o_per.reshape(-1).tolist()


def test_pages_bytes_known_totals():
    """Stored pages: tiny 16 + 9; Mistral-shaped 128 + 7 x 25; Qwen3-shaped 1024 + 7 x 97; a mixed
    DeepSeek-style layer 8 x 1024 + 56 x 65 (hand-derived from the storage rule)."""
    expect = {"tiny": 25, "mistral-7b": 303, "qwen3-32b": 1703, "dsv4-flash-l3": 11832, "dsv4-flash-l0": 65536}
    for name, w, layer in _all_layer_cases():
        if name not in expect:
            continue
        dims = sp.Dims(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, w.page_size)
        _, _, per = sp.segpaged_pages_bytes(dims, w.ctx_lens, w.q_lens, w.classes[layer])
        assert int(per.sum()) == expect[name], name


EDGE = [
    # (seqs [(L, Lq)], Hq, Hkv, D, P, classes [B][Hkv])
    ([(256, 64)], 4, 2, 64, 16, [[(1, 0, 0), (0, 4, 64)]]),
    ([(1000, 300), (37, 37), (5, 0), (129, 1)], 8, 2, 128, 32, [[(0, 0, 100), (1, 0, 0)], [(0, 50, 3), (0, 2, 1)], [(1, 0, 0), (0, 1, 1)], [(0, 128, 1), (1, 0, 0)]]),
    ([(300, 300)], 8, 8, 64, 128, [[(0, 5, 17), (0, 0, 1), (1, 0, 0), (0, 300, 300), (0, 1000, 2), (0, 64, 64), (0, 127, 129), (0, 3, 250)]]),
    ([(777, 200)], 16, 2, 128, 16, [[(0, 16, 16), (0, 17, 15)]]),
    ([(4100, 1030)], 2, 2, 128, 64, [[(0, 64, 1024), (1, 0, 0)]]),
]


def _units_cover_exactly(w_seqs, Hq, Hkv, D, P, classes, split_ctas=0):
    """Every (query row, head) of every sequence is run by exactly one unit, over KV tiles that together
    hold every key the oracle says the row can see; chunks of a split unit tile its KV range exactly and
    each combine record names its chunks' partial slots."""
    B = len(w_seqs)
    dims = sp.Dims(B, Hq, Hkv, D, P)
    ctx = [s[0] for s in w_seqs]
    ql = [s[1] for s in w_seqs]
    cls = np.asarray(classes, np.int32)
    _, _, per = sp.segpaged_pages_bytes(dims, ctx, ql, cls)
    offs = np.concatenate([[0], np.cumsum(per)]).astype(np.int32)
    recs, info = sp.segpaged_prefill_plan(dims, ctx, ql, cls, offs, split_ctas)
    nu, ng = info["num_units"], info["num_groups"]
    assert len(recs) == nu + ng
    units, groups = recs[:nu], recs[nu:]
    G = Hq // Hkv
    cu_q = np.concatenate([[0], np.cumsum(ql)])
    seen = np.zeros((int(cu_q[-1]), Hkv), np.int32)
    ppt = 128 // P
    cost = [int(u[U_NTILES]) * (1 if u[U_HALF] else 2) for u in units]
    max_cost = max(cost + [1])
    prev = 1 << 30
    chunks = {}
    for u, c in zip(units, cost):
        bucket = (c * 16 + max_cost // 2) // max_cost
        assert bucket <= prev  # longest first, by cost bucket
        prev = bucket
        b, kh = int(u[U_SEQ]), int(u[U_KVH])
        L, Lq = ctx[b], ql[b]
        g, S, W = (int(x) for x in cls[b, kh])
        stored = orc.stored_logical_pages(L, Lq, bool(g), S, W, P)
        assert u[U_TOTAL] == len(stored) and u[U_TOFF] == offs[b * Hkv + kh]
        npages = int(u[U_AN] + u[U_BN])
        n_kv = -(-npages // ppt)
        assert 0 <= u[U_T0] and u[U_T0] + u[U_NTILES] <= n_kv and u[U_NTILES] >= 1
        idxs = [x if x < u[U_AN] else int(u[U_B0]) + x - int(u[U_AN]) for x in range(npages)]
        assert len(set(idxs)) == npages and all(0 <= x < len(stored) for x in idxs)
        lps = [x if x < u[U_NSINK] else int(u[U_W0]) + x - int(u[U_NSINK]) for x in idxs]
        assert lps == [stored[x] for x in idxs]          # table index -> logical page is the storage order
        assert 1 <= u[U_NPOS] <= 256 // G and u[U_HALF] == (u[U_NPOS] <= 128 // G)
        key = (b, kh, int(u[U_QROW]))
        if u[U_PART] >= 0:
            chunks.setdefault(key, []).append((int(u[U_T0]), int(u[U_NTILES]), int(u[U_PART])))
            continue
        assert u[U_T0] == 0 and u[U_NTILES] == n_kv
        covered = set()
        for lp in lps:
            covered.update(range(lp * P, lp * P + P))
        for r in range(int(u[U_NPOS])):
            i = int(u[U_POS0]) + r
            row = int(u[U_QROW]) + r
            assert row - cu_q[b] == i - (L - Lq)
            assert set(orc.visible_keys(bool(g), S, W, i).tolist()) <= covered
            seen[row, kh] += 1
    slots = set()
    for grp in groups:
        b, kh = int(grp[U_SEQ]), int(grp[U_KVH])
        key = (b, kh, int(grp[U_QROW]))
        parts = sorted(chunks.pop(key))
        assert len(parts) == grp[U_NSPLIT] >= 2
        assert [p[2] for p in parts] == list(range(int(grp[U_PART]), int(grp[U_PART] + grp[U_NSPLIT])))
        t = 0
        for t0, n, _ in parts:                           # chunks tile the unit's KV range in order
            assert t0 == t
            t += n
        npages = int(grp[U_AN] + grp[U_BN])
        assert t == -(-npages // ppt)
        slots.update(p[2] for p in parts)
        for r in range(int(grp[U_NPOS])):
            seen[int(grp[U_QROW]) + r, kh] += 1
    assert not chunks and len(slots) == info["num_partials"]
    assert np.all(seen == 1)
    # the combine grid reaches the last valid row of every record: row of position p, head h is
    # (p // (128/G)) * 128 + (p % (128/G)) * G + h; a block per 32 rows
    npt = 128 // G
    need = 0
    for grp in groups:
        last = max((p // npt) * 128 + (p % npt) * G + G - 1 for p in range(int(grp[U_NPOS]))) + 1
        need = max(need, -(-last // 32))
    assert info["combine_row_blocks"] == need
    assert info["num_half_units"] == sum(int(u[U_HALF]) for u in units)
    return units


@pytest.mark.parametrize("case", range(len(EDGE)))
def test_plan_units_cover_every_row_once_and_every_visible_key(case):
    _units_cover_exactly(*EDGE[case])


@pytest.mark.parametrize("case", range(len(EDGE)))
def test_plan_with_splits_covers_every_row_once(case):
    _units_cover_exactly(*EDGE[case], split_ctas=1000)


def _random_shapes(n, seed):
    """Seeded random small layers: 1-3 sequences of up to 800 tokens (some with empty or whole-sequence query
    ranges), G in {1, 2, 4, 8, 16}, D in {64, 128}, P in {16, 32, 64, 128}, and per (sequence, KV head) a global
    head or a local one with a random sink (0 up to past the end) and window (1 up to past the end)."""
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(n):
        B = int(rng.integers(1, 4))
        seqs = []
        for _ in range(B):
            L = int(rng.integers(1, 801))
            Lq = int(rng.choice([0, 1, L, int(rng.integers(0, L + 1))]))
            seqs.append((L, Lq))
        Hkv = int(rng.integers(1, 4))
        G = int(rng.choice([1, 2, 4, 8, 16]))
        D = int(rng.choice([64, 128]))
        P = int(rng.choice([16, 32, 64, 128]))
        classes = [[(1, 0, 0) if rng.random() < 0.3 else (0, int(rng.integers(0, 300)), int(rng.integers(1, 900)))
                    for _ in range(Hkv)] for _ in range(B)]
        split = int(rng.choice([0, 148, 1000]))
        out.append((seqs, Hkv * G, Hkv, D, P, classes, split))
    return out


@pytest.mark.parametrize("case", range(24))
def test_plan_covers_every_row_once_on_random_shapes(case):
    """The planner's exact-cover and visible-key properties (as on the edge shapes) on seeded random layers,
    with and without splitting."""
    seqs, Hq, Hkv, D, P, classes, split = _random_shapes(24, 20251203)[case]
    _units_cover_exactly(seqs, Hq, Hkv, D, P, classes, split_ctas=split)


def test_split_policy_on_workloads():
    """Long-context prefill is never split; decode-like tiles and the 8K layer are."""
    def plan(w):
        dims = sp.Dims(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, w.page_size)
        _, _, per = sp.segpaged_pages_bytes(dims, w.ctx_lens, w.q_lens, w.classes[0])
        offs = np.concatenate([[0], np.cumsum(per)]).astype(np.int32)
        return sp.segpaged_prefill_plan(dims, w.ctx_lens, w.q_lens, w.classes[0], offs, 148)
    for name in ("qwen3-32b", "llama-3.3-70b"):
        assert plan(synth.get(name))[1]["num_groups"] == 0, name
    assert plan(synth.dsv4_flash(layers=4))[1]["num_groups"] == 0
    for name in ("qwen3-32b-lq16", "qwen3-32b-lq64", "mistral-7b"):
        recs, i = plan(synth.get(name))
        work = recs[:i["num_units"]]
        cost = work[:, U_NTILES].astype(np.int64) * np.where(work[:, U_HALF] == 1, 1, 2)
        share = -(-int(cost.sum()) // 148)                 # one CTA's share of the tensor work
        assert i["num_groups"] > 0, name
        assert cost.max() <= max(share, 16) + 2, (name, int(cost.max()), share)   # about one wave of equal pieces


def test_noalloc_refuses_split_plans():
    """Checked on the host before any device work."""
    w = synth.get("qwen3-32b-lq16")
    dims = sp.Dims(1, 64, 8, 128, 128, 2000)
    _, _, per = sp.segpaged_pages_bytes(dims, w.ctx_lens, w.q_lens, w.classes[0])
    offs = np.concatenate([[0], np.cumsum(per)]).astype(np.int32)
    recs, info = sp.segpaged_prefill_plan(dims, w.ctx_lens, w.q_lens, w.classes[0], offs, 148)
    recs = np.ascontiguousarray(recs)
    rc = sp.library().segpaged_attn_prefill_noalloc(ctypes.byref(dims.c()), None, 16, None, None, None, 0,
                                                     recs.ctypes.data_as(ctypes.c_void_p), len(recs), 0.1, None, None,
                                                     None, None)
    assert rc == -9


def test_prefill_rejects_a_plan_made_for_another_call():
    """A plan records the shape of the call it was made for (rows, heads, head_dim, page size, page-table
    length); a call that disagrees gets SEGPAGED_ERR_DIMS before anything is enqueued, and the allocation-free
    entry point checks every unit of its host plan the same way. Only calls the host checks refuse are made
    here: the device addresses are fake (aligned, never dereferenced)."""
    dims = sp.Dims(2, 8, 2, 64, 16, 4000)
    ctx, ql = [900, 300], [200, 64]
    cls = [[(1, 0, 0), (0, 4, 64)], [(0, 8, 100), (1, 0, 0)]]
    _, _, per = sp.segpaged_pages_bytes(dims, ctx, ql, cls)
    offs = np.concatenate([[0], np.cumsum(per)]).astype(np.int32)
    units, info = sp.segpaged_prefill_plan(dims, ctx, ql, cls, offs, 0)
    assert info["total_q"] == 264 and info["page_table_len"] == int(offs[-1])
    assert (info["num_q_heads"], info["num_kv_heads"], info["head_dim"], info["page_size"]) == (8, 2, 64, 16)
    lib = sp.library()
    fake = ctypes.c_void_p(1 << 24)

    def prefill(d, total_q, table_len, inf):
        return lib.segpaged_attn_prefill(ctypes.byref(d.c()), fake, total_q, fake, fake, fake, table_len, fake,
                                         ctypes.byref(sp._info(inf)), 0.125, fake, fake, fake, 1 << 26, None, None)

    # the plan of a longer query range (264 rows) given to a call with fewer rows, or more
    assert prefill(dims, 200, int(offs[-1]), info) == -2
    assert prefill(dims, 300, int(offs[-1]), info) == -2
    # a page table shorter than the entries the plan addresses
    assert prefill(dims, 264, int(offs[-1]) - 1, info) == -2
    # other head counts, head_dim or page size than the plan's
    for other in (sp.Dims(2, 16, 2, 64, 16, 4000), sp.Dims(2, 8, 4, 64, 16, 4000), sp.Dims(2, 8, 2, 128, 16, 4000),
                  sp.Dims(2, 8, 2, 64, 32, 4000)):
        assert prefill(other, 264, int(offs[-1]), info) == -2
    # an info that disagrees with itself: half units beyond the units, combine records without partial slots
    assert prefill(dims, 264, int(offs[-1]), dict(info, num_half_units=info["num_units"] + 1)) == -2
    assert prefill(dims, 264, int(offs[-1]), dict(info, num_groups=1, num_partials=0)) == -2
    # the same rules through the other prefill entry points
    assert lib.segpaged_attn_prefill_append(ctypes.byref(dims.c()), fake, 200, fake, fake, fake, fake, fake,
                                            int(offs[-1]), fake, ctypes.byref(sp._info(info)), 0.125, fake, fake, fake,
                                            1 << 26, None, None) == -2
    assert lib.segpaged_attn_prefill_rope(ctypes.byref(dims.c()), fake, 200, fake, fake, fake, int(offs[-1]), fake,
                                          ctypes.byref(sp._info(info)), 0.125, fake, fake, fake, fake, fake, fake,
                                          1 << 26, None, None) == -2

    # allocation-free entry point: every unit is checked against the call's rows, heads and table
    def noalloc(recs, total_q, table_len, d=dims):
        recs = np.ascontiguousarray(recs, dtype=np.int32)
        return lib.segpaged_attn_prefill_noalloc(ctypes.byref(d.c()), fake, total_q, fake, fake, fake, table_len,
                                                 recs.ctypes.data_as(ctypes.c_void_p), len(recs), 0.125, fake, fake,
                                                 None, None)

    U_QROW, U_KVH, U_TOFF = 0, 3, 4
    assert noalloc(units, 200, int(offs[-1])) == -2                     # rows past the call's 200
    assert noalloc(units, 264, int(offs[-1]) - 1) == -2                 # entries past the call's table
    assert noalloc(units, 264, int(offs[-1]), sp.Dims(2, 8, 1, 64, 16, 4000)) == -2   # KV head 1 of 1
    for field, value in ((U_QROW, -1), (U_KVH, 2), (U_KVH, -1), (U_TOFF, -3)):
        bad = units.copy()
        bad[len(bad) // 2, field] = value
        assert noalloc(bad, 264, int(offs[-1])) == -2, (field, value)


@pytest.mark.parametrize("name", ["tiny", "mistral-7b", "llama-3.3-70b", "qwen3-32b"])
def test_plan_workloads(name):
    w = synth.get(name)
    seqs = list(zip(w.ctx_lens, w.q_lens))
    if name in ("llama-3.3-70b", "qwen3-32b"):       # the set checks are slow in Python at full size
        seqs = [(min(L, 9000), min(Lq, 700)) for L, Lq in seqs]
    _units_cover_exactly(seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, w.page_size, w.classes[0].tolist())


def test_rope_table_matches_oracle():
    deltas = list(range(4096))
    for D in (64, 128):
        got = sp.segpaged_rope_cos_sin(1e6, deltas, D)
        want = orc.rope_cos_sin(1e6, deltas, D)
        np.testing.assert_array_equal(got, want)


def test_validation_errors():
    dims = sp.Dims(1, 4, 2, 64, 16)
    with pytest.raises(sp.SegPagedError) as e:
        sp.segpaged_pages_bytes(sp.Dims(1, 4, 2, 96, 16), [10], [5], [[1, 0, 0], [1, 0, 0]])
    assert e.value.code == -2
    with pytest.raises(sp.SegPagedError) as e:
        sp.segpaged_pages_bytes(sp.Dims(1, 4, 3, 64, 16), [10], [5], [[1, 0, 0]] * 3)
    assert e.value.code == -2
    with pytest.raises(sp.SegPagedError) as e:
        sp.segpaged_pages_bytes(sp.Dims(1, 4, 2, 64, 24), [10], [5], [[1, 0, 0], [1, 0, 0]])
    assert e.value.code == -2
    with pytest.raises(sp.SegPagedError) as e:
        sp.segpaged_pages_bytes(dims, [10], [11], [[1, 0, 0], [1, 0, 0]])
    assert e.value.code == -4
    with pytest.raises(sp.SegPagedError) as e:
        sp.segpaged_pages_bytes(dims, [10], [5], [[1, 0, 0], [0, 4, 0]])
    assert e.value.code == -3
    # page-table offsets that disagree with the storage rule
    with pytest.raises(sp.SegPagedError) as e:
        sp.segpaged_prefill_plan(dims, [256], [64], [[1, 0, 0], [0, 4, 64]], [0, 16, 24])
    assert e.value.code == -5
    lib = sp.library()
    # NULL dims and NULL arrays
    assert lib.segpaged_pages_bytes(None, None, None, None, None, None) == -1
    info = sp._PlanInfo(3, 0, 0)
    assert lib.segpaged_attn_prefill(ctypes.byref(dims.c()), None, 1, None, None, None, 0, None, ctypes.byref(info), 1.0,
                                     None, None, None, 256, None, None) == -1
    assert lib.segpaged_build(ctypes.byref(dims.c()), *([None] * 12)) == -1
    assert sp.error_string(-5).startswith("page-table")


# Mass item field positions (head_sparse_paged_b200/csrc/mass_sm100.cuh).
(M_SEQ, M_KVH, M_TILE, M_TOFF, M_NSINK, M_W0, M_GLOBAL, M_SINK, M_WIN, M_Q0, M_L, M_QROW0, M_T0, M_NT, M_TOTAL,
 M_LQ) = range(16)


@pytest.mark.parametrize("case", range(len(EDGE)))
def test_mass_plan_covers_every_query_key_and_every_viewer(case):
    """Each (sequence, KV head) gets one item per 128-key tile that holds a key of the query range;
    an item's query tiles [t0, t0 + nt) include every query tile with a row that sees one of those
    keys (the oracle's visibility rule) and start and end on such tiles; the key pages it reads are
    stored, at the table index the storage order gives; items come longest first."""
    _mass_plan_check(*EDGE[case])


@pytest.mark.parametrize("case", range(12))
def test_mass_plan_on_random_shapes(case):
    seqs, Hq, Hkv, D, P, classes, _ = _random_shapes(12, 20251204)[case]
    _mass_plan_check(seqs, Hq, Hkv, D, P, classes)


def _mass_plan_check(w_seqs, Hq, Hkv, D, P, classes):
    B = len(w_seqs)
    dims = sp.Dims(B, Hq, Hkv, D, P)
    ctx = [s[0] for s in w_seqs]
    ql = [s[1] for s in w_seqs]
    cls = np.asarray(classes, np.int32)
    _, _, per = sp.segpaged_pages_bytes(dims, ctx, ql, cls)
    offs = np.concatenate([[0], np.cumsum(per)]).astype(np.int32)
    items = sp.segpaged_mass_plan(dims, ctx, ql, cls, offs)
    G = Hq // Hkv
    npos = 128 // G
    cu_q = np.concatenate([[0], np.cumsum(ql)])
    nts = [int(it[M_NT]) for it in items]
    assert nts == sorted(nts, reverse=True)
    got = {}
    for it in items:
        b, kh, x = int(it[M_SEQ]), int(it[M_KVH]), int(it[M_TILE])
        assert (b, kh, x) not in got
        got[(b, kh, x)] = it
        L, Lq = ctx[b], ql[b]
        q0 = L - Lq
        g, S, W = (int(v) for v in cls[b, kh])
        assert (it[M_Q0], it[M_L], it[M_LQ], it[M_QROW0]) == (q0, L, Lq, cu_q[b])
        assert it[M_TOFF] == offs[b * Hkv + kh]
        stored = orc.stored_logical_pages(L, Lq, bool(g), S, W, P)
        assert it[M_TOTAL] == len(stored)
        for c in range(128 // P):            # pages with a key of the query range are stored, at their index
            lp = x * (128 // P) + c
            if lp * P + P <= q0 or lp * P >= L:
                continue
            idx = lp if g else (lp if lp < it[M_NSINK] else int(it[M_NSINK]) + lp - int(it[M_W0]))
            assert stored[idx] == lp
        viewers = set()
        jmin, jmax = max(q0, 128 * x), min(L, 128 * x + 128) - 1
        for i in range(q0, L):
            v = orc.visible_keys(bool(g), S, W, i)
            at = int(np.searchsorted(v, jmin))
            if at < len(v) and v[at] <= jmax:
                viewers.add((i - q0) // npos)
        t0, nt = int(it[M_T0]), int(it[M_NT])
        assert viewers <= set(range(t0, t0 + nt))
        assert t0 in viewers and t0 + nt - 1 in viewers
    for b in range(B):
        L, Lq = ctx[b], ql[b]
        for kh in range(Hkv):
            want = set(range((L - Lq) // 128, (L - 1) // 128 + 1)) if Lq > 0 else set()
            assert {x for (bb, k, x) in got if bb == b and k == kh} == want


# Append-mode fields (head_sparse_paged_b200/csrc/plan.h).
U_NOLDT, U_NEW0, U_NNEW, U_SPLITQ, U_CUQ = 20, 21, 22, 23, 24


@pytest.mark.parametrize("case", range(len(EDGE)))
@pytest.mark.parametrize("split", [0, 1000])
def test_append_plan_reads_old_keys_from_pool_and_new_keys_fresh(case, split):
    """Fused append-and-attend plan: a unit's page list holds only pages with a key before q0; its new pages
    (read from the new K/V) are consecutive logical pages from the first visible key at or after q0 to its
    last row; together they hold every visible key of every row (the oracle's sets); rows are covered once."""
    _append_plan_check(*EDGE[case], split)


@pytest.mark.parametrize("case", range(12))
def test_append_plan_on_random_shapes(case):
    seqs, Hq, Hkv, D, P, classes, split = _random_shapes(12, 20251205)[case]
    _append_plan_check(seqs, Hq, Hkv, D, P, classes, split)


def _append_plan_check(w_seqs, Hq, Hkv, D, P, classes, split):
    B = len(w_seqs)
    dims = sp.Dims(B, Hq, Hkv, D, P)
    ctx = [s[0] for s in w_seqs]
    ql = [s[1] for s in w_seqs]
    cls = np.asarray(classes, np.int32)
    _, _, per = sp.segpaged_pages_bytes(dims, ctx, ql, cls)
    offs = np.concatenate([[0], np.cumsum(per)]).astype(np.int32)
    recs, info = sp.segpaged_prefill_plan_append(dims, ctx, ql, cls, offs, split)
    units = recs[: info["num_units"]]
    cu_q = np.concatenate([[0], np.cumsum(ql)])
    ppt = 128 // P
    seen = np.zeros((int(cu_q[-1]), Hkv), np.int32)
    for u in units:
        b, kh = int(u[U_SEQ]), int(u[U_KVH])
        L, Lq = ctx[b], ql[b]
        q0 = L - Lq
        g, S, W = (int(x) for x in cls[b, kh])
        assert u[U_SPLITQ] == q0 and u[U_CUQ] == cu_q[b]
        npages = int(u[U_AN] + u[U_BN])
        assert u[U_NOLDT] == -(-npages // ppt)
        assert u[U_NTILES] == u[U_NOLDT] + -(-int(u[U_NNEW]) // ppt) or u[U_PART] >= 0
        stored = orc.stored_logical_pages(L, Lq, bool(g), S, W, P)
        idxs = [x if x < u[U_AN] else int(u[U_B0]) + x - int(u[U_AN]) for x in range(npages)]
        lps = [x if x < u[U_NSINK] else int(u[U_W0]) + x - int(u[U_NSINK]) for x in idxs]
        assert lps == [stored[x] for x in idxs]
        assert all(lp * P < q0 for lp in lps)
        new = list(range(int(u[U_NEW0]), int(u[U_NEW0]) + int(u[U_NNEW])))
        covered_old = set()
        for lp in lps:
            covered_old.update(range(lp * P, lp * P + P))
        covered_new = set()
        for lp in new:
            covered_new.update(range(lp * P, lp * P + P))
        if u[U_PART] >= 0 and u[U_T0] != 0:
            continue
        for r in range(int(u[U_NPOS])):
            i = int(u[U_POS0]) + r
            vis = set(orc.visible_keys(bool(g), S, W, i).tolist())
            assert {j for j in vis if j < q0} <= covered_old
            assert {j for j in vis if j >= q0} <= covered_new
            seen[int(u[U_QROW]) + r, kh] += 1
        if new:
            last = int(u[U_POS0]) + int(u[U_NPOS]) - 1
            assert new[-1] == last // P
            first_vis = min(j for r in range(int(u[U_NPOS])) for j in orc.visible_keys(bool(g), S, W, int(u[U_POS0]) + r)
                            if j >= q0)
            assert new[0] == first_vis // P
    assert np.all(seen == 1)


def test_binding_rejects_tensors_off_the_current_device(monkeypatch):
    """The library launches on the current device, so the binding refuses a tensor on another one before
    any call (checked with a stand-in tensor: this machine has no GPU)."""
    class FakeCudaTensor:
        is_cuda = True
        dtype = torch.bfloat16

        def __init__(self, index):
            self.device = torch.device("cuda", index)

        def is_contiguous(self):
            return True

        def data_ptr(self):
            return 4096

    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    with pytest.raises(ValueError, match="current device is cuda:0"):
        sp._dev(FakeCudaTensor(1), torch.bfloat16, "q")
    assert sp._dev(FakeCudaTensor(0), torch.bfloat16, "q").value == 4096


def test_visible_flops_match_hand_count_and_enumeration():
    """The reported metric's numerator, 4 * D * sum |V(i)| over (query row, query head), against the tiny
    layer counted by hand (global rows 192..255 see i + 1 keys; local rows see 4 sink + 64 window keys, which
    do not meet) and against the oracle's explicit visible sets on ragged shapes."""
    from head_sparse_paged_b200.counts import visible_flops
    w = synth.tiny()
    assert visible_flops(w) == 4 * 64 * 2 * (sum(range(193, 257)) + 64 * (4 + 64))
    assert abs(visible_flops(w) / 1e12 - 9.6e-6) < 0.05e-6          # the tiny configuration's figure
    w = synth.custom("ragged", [(1000, 300), (37, 37), (5, 0), (129, 1), (300, 300)], 8, 2, 64, 16,
                     [[(0, 0, 100), (1, 0, 0)], [(0, 50, 3), (0, 2, 1)], [(1, 0, 0), (0, 1, 1)],
                      [(0, 128, 1), (1, 0, 0)], [(0, 1000, 2), (0, 127, 129)]], seed=7)
    want = 0
    for b, (L, Lq) in enumerate(zip(w.ctx_lens, w.q_lens)):
        for kh in range(w.num_kv_heads):
            g, S, W = (int(x) for x in w.classes[0, b, kh])
            want += sum(len(orc.visible_keys(bool(g), S, W, i)) for i in range(L - Lq, L))
    assert visible_flops(w) == 4 * 64 * w.group * want


def test_mass_pair_count_matches_enumeration():
    """The token-mass leg's work count (one exponential per visible (query row, query head, key of the query
    range)) against the oracle's explicit visible sets."""
    from head_sparse_paged_b200.counts import mass_pairs
    w = synth.custom("ragged", [(1000, 300), (37, 37), (5, 0), (129, 1), (300, 300)], 8, 2, 64, 16,
                     [[(0, 0, 100), (1, 0, 0)], [(0, 50, 3), (0, 2, 1)], [(1, 0, 0), (0, 1, 1)],
                      [(0, 128, 1), (1, 0, 0)], [(0, 1000, 2), (0, 127, 129)]], seed=7)
    want = 0
    for b, (L, Lq) in enumerate(zip(w.ctx_lens, w.q_lens)):
        for kh in range(w.num_kv_heads):
            g, S, W = (int(x) for x in w.classes[0, b, kh])
            want += sum(int((orc.visible_keys(bool(g), S, W, i) >= L - Lq).sum()) for i in range(L - Lq, L))
    assert mass_pairs(w, 0) == w.group * want


def test_rope_path_choice():
    """The caller-level RoPE path: re-alignment pass when a (sequence, KV head) has more than one work unit of
    2 x 128 / G positions, gather-time rotation otherwise."""
    from head_sparse_paged_b200.runner import rope_realign_preferred
    assert not rope_realign_preferred([16] * 32, 8)          # decode-like batch: one unit per head
    assert not rope_realign_preferred([32, 5], 8)            # exactly one unit of 2 x 16 positions
    assert rope_realign_preferred([33], 8)
    assert rope_realign_preferred([4096], 1)                 # 43-layer workload: 16 units per head
    assert not rope_realign_preferred([256], 1) and rope_realign_preferred([257], 1)
    assert not rope_realign_preferred([], 4)
