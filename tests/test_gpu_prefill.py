"""segpaged_attn_prefill on the GPU against the fp64 oracle.

Small and mid-size shapes are compared on every output row; the full-size layer workloads on
sampled rows (all query heads of each sampled row), computed one by one by the oracle from the
unpaged dense inputs. Tolerances: gpu_common.O_TOL / LSE_TOL.
"""
import math

import numpy as np
import pytest
import torch

from head_sparse_paged_b200 import synth
from head_sparse_paged_b200.runner import Runner
from oracle import reference as orc

from gpu_common import compare, full_problem, head_problem, oracle_dense, sample_rows

pytestmark = pytest.mark.gpu

_LIB = None


def lib():
    global _LIB
    if _LIB is None:
        _LIB = orc.OracleLib()
    return _LIB


def _run(w, **kw):
    kw.setdefault("keep_dense", True)
    r = Runner(w, **kw)
    r.step()
    torch.cuda.synchronize()
    r.check_status()
    return r


SMALL = {
    "tiny": lambda: synth.tiny(),
    "mistral-7b": lambda: synth.mistral_7b(),
    # several sequences, ragged tails, an empty query range, W < P, S > L, Lq = L, Lq = 1, G = 4
    "varlen-p16-g4": lambda: synth.custom("varlen-p16-g4", [(1000, 300), (37, 37), (5, 0), (129, 1), (700, 129)], 8, 2,
                                          128, 16, [[(0, 0, 100), (1, 0, 0)], [(0, 50, 3), (0, 2, 1)],
                                                    [(1, 0, 0), (0, 1, 1)], [(0, 128, 1), (1, 0, 0)],
                                                    [(0, 17, 200), (0, 1, 31)]], seed=21),
    # MHA (G = 1), D = 64, P = 128, every class corner, two sequences
    "mha-d64-p128": lambda: synth.custom("mha-d64-p128", [(300, 300), (1300, 260)], 8, 8, 64, 128,
                                         [[(0, 5, 17), (0, 0, 1), (1, 0, 0), (0, 300, 300), (0, 1000, 2), (0, 64, 64),
                                           (0, 127, 129), (0, 3, 250)]] * 2, seed=22, page_order="interleaved"),
    # G = 8 and G = 16 packing (16 and 8 positions per tile), P = 32 and P = 64
    "g8-p32": lambda: synth.custom("g8-p32", [(2000, 333)], 16, 2, 128, 32, [[(1, 0, 0), (0, 64, 256)]], seed=23),
    "g16-p64": lambda: synth.custom("g16-p64", [(1500, 77), (64, 64)], 32, 2, 64, 64,
                                    [[(0, 0, 64), (1, 0, 0)], [(0, 64, 1), (0, 3, 5)]], seed=24),
    # G = 2, D = 128, window a multiple of the tile, sink ending inside a page
    "g2-p64": lambda: synth.custom("g2-p64", [(4100, 1030)], 4, 2, 128, 64, [[(0, 70, 1024), (1, 0, 0)]], seed=25,
                                   rope_theta=1e6, rope_deltas=[1234]),
}


SPLIT = {
    # decode-like query ranges over long contexts: the planner splits the long units across CTAs
    "split-short-q": (lambda: synth.custom("split-short-q", [(3000, 7), (5000, 1), (700, 40), (2500, 130)], 8, 2, 128,
                                           64, [[(1, 0, 0), (0, 64, 512)], [(0, 0, 300), (1, 0, 0)],
                                                [(1, 0, 0), (1, 0, 0)], [(0, 16, 1000), (1, 0, 0)]], seed=31), None),
    "qwen3-32b-lq16": (lambda: synth.get("qwen3-32b-lq16"), None),
    "qwen3-32b-lq64": (lambda: synth.get("qwen3-32b-lq64"), None),
    # splits forced on the edge shapes (every unit longer than 8 KV tiles is cut)
    "varlen-p16-g4-forced": (lambda: synth.custom("varlen-p16-g4-forced", [(2000, 300), (37, 37), (5, 0), (900, 129)],
                                                  8, 2, 128, 16, [[(0, 0, 100), (1, 0, 0)], [(0, 50, 3), (0, 2, 1)],
                                                                  [(1, 0, 0), (0, 1, 1)], [(0, 17, 200), (0, 1, 31)]],
                                                  seed=32), 1000),
    "mha-d64-p128-forced": (SMALL["mha-d64-p128"], 1000),
    "g2-p64-forced": (SMALL["g2-p64"], 1000),
    # a decode-like batch: every unit a half unit (the variant with the second query buffer as a K/V slot)
    "llama-decode8x16": (lambda: synth.llama_70b_decode(8, 16), None),
}


def _every_row(name, w, r):
    st = r.state[0]
    k, v = r.dense[0]
    qn, kn, vn = oracle_dense(w, st.q, k, v)
    pb = full_problem(w, 0, qn, kn, vn)
    items = np.array([(row, h) for row in range(w.total_q) for h in range(w.num_q_heads)], np.int64)
    o_ref, lse_ref = lib().attention(pb, r.scale, items)
    o = st.o.float().cpu().numpy().reshape(-1, w.head_dim)
    lse = st.lse.cpu().numpy().T.reshape(-1)
    compare(o, lse, o_ref, lse_ref, name)


@pytest.mark.parametrize("name", list(SPLIT))
def test_split_prefill_matches_oracle_every_row(name):
    make, split = SPLIT[name]
    w = make()
    r = _run(w, split_ctas=split)
    assert r.state[0].info["num_groups"] > 0, "expected a split plan"
    _every_row(name, w, r)


def test_combine_grid_too_small_sets_status():
    """A plan info whose combine_row_blocks is below what the plan needs leaves rows unmerged; the
    combine launch reports it in the status word (SEGPAGED_STATUS_UNIT) instead of failing silently."""
    w = SPLIT["split-short-q"][0]()
    r = _run(w)
    info = r.state[0].info
    assert info["combine_row_blocks"] > 1
    info["combine_row_blocks"] = 1
    r.prefill(0)
    torch.cuda.synchronize()
    assert int(r.status.item()) & 8
    r.status.zero_()


def test_split_prefill_is_bit_identical_under_page_permutation():
    w = SPLIT["split-short-q"][0]()
    a = _run(w)
    b = _run(w, page_seed_offset=7)
    assert torch.equal(a.state[0].o, b.state[0].o) and torch.equal(a.state[0].lse, b.state[0].lse)


@pytest.mark.parametrize("name", list(SMALL))
def test_prefill_matches_oracle_every_row(name):
    w = SMALL[name]()
    r = _run(w)
    st = r.state[0]
    k, v = r.dense[0]
    qn, kn, vn = oracle_dense(w, st.q, k, v)
    pb = full_problem(w, 0, qn, kn, vn)
    items = np.array([(row, h) for row in range(w.total_q) for h in range(w.num_q_heads)], np.int64)
    o_ref, lse_ref = lib().attention(pb, r.scale, items)
    o = st.o.float().cpu().numpy().reshape(-1, w.head_dim)
    lse = st.lse.cpu().numpy().T.reshape(-1)
    compare(o, lse, o_ref, lse_ref, name)


def test_prefill_is_bit_identical_under_page_permutation():
    w = SMALL["varlen-p16-g4"]()
    a = _run(w)
    b = _run(w, page_seed_offset=99)
    assert not np.array_equal(a.state[0].table, b.state[0].table)
    assert torch.equal(a.state[0].o, b.state[0].o)
    assert torch.equal(a.state[0].lse, b.state[0].lse)


def test_prefill_is_deterministic_across_calls():
    w = synth.mistral_7b()
    r = _run(w)
    o1, l1 = r.state[0].o.clone(), r.state[0].lse.clone()
    r.step()
    torch.cuda.synchronize()
    assert torch.equal(o1, r.state[0].o) and torch.equal(l1, r.state[0].lse)


@pytest.mark.parametrize("name", ["varlen-p16-g4", "mha-d64-p128"])
def test_prefill_output_only_16_byte_aligned(name):
    """O at an address that is 16- but not 32-byte aligned takes the epilogue's 16-byte stores; the result must be
    the 32-byte-store path's bit for bit."""
    from head_sparse_paged_b200 import segpaged as sp
    w = SMALL[name]()
    r = _run(w)
    st = r.state[0]
    buf = torch.full((st.o.numel() + 32,), float("nan"), dtype=torch.bfloat16, device=st.o.device)
    base = (-(buf.data_ptr() // 2)) % 16                  # elements to the next 32-byte boundary
    o = buf[base + 8: base + 8 + st.o.numel()].view(st.o.shape)
    assert o.data_ptr() % 32 == 16
    lse = torch.full_like(st.lse, float("nan"))
    sp.segpaged_attn_prefill(r.dims, st.q, r.k_pool, r.v_pool, st.table_dev, st.units_dev, st.info, r.scale, o, lse,
                             r.workspace, r.status)
    torch.cuda.synchronize()
    r.check_status()
    assert st.o.data_ptr() % 32 == 0
    assert torch.equal(o, st.o) and torch.equal(lse, st.lse)


FULL = {
    "llama-3.3-70b": lambda: (synth.llama_70b(), [0]),
    "llama-3.3-70b-2-globals": lambda: (synth.llama_70b(globals_per_seq=2), [0]),
    "qwen3-32b": lambda: (synth.qwen3_32b(), [0]),
    "dsv4-flash-all-global-and-mixed": lambda: (synth.dsv4_flash(), [0, 3]),
}


@pytest.mark.parametrize("name", list(FULL))
def test_prefill_full_size_sampled(name):
    w, layers = FULL[name]()
    r = _run(w, layers=layers)
    rng = np.random.default_rng(5)
    G = w.group
    npos = 128 // G
    for li in layers:
        st = r.state[li]
        k, v = r.dense[li]
        o_all = st.o
        lse_all = st.lse
        heads = range(w.num_kv_heads) if w.num_kv_heads <= 8 else sorted(rng.choice(w.num_kv_heads, 8, replace=False))
        for b in range(w.num_seqs):
            for kh in heads:
                pb = head_problem(w, li, b, int(kh), st.q, k, v)
                rows = sample_rows(w.q_lens[b], npos, rng, extra=3)
                items = np.array([(row, h) for row in rows for h in range(G)], np.int64)
                o_ref, lse_ref = lib().attention(pb, r.scale, items)
                gr = torch.tensor([int(w.cu_q()[b]) + row for row in rows for _ in range(G)], device=o_all.device)
                gh = torch.tensor([int(kh) * G + h for _ in rows for h in range(G)], device=o_all.device)
                o = o_all[gr, gh].float().cpu().numpy()
                lse = lse_all[gh, gr].cpu().numpy()
                compare(o, lse, o_ref, lse_ref, f"{name} layer {li} seq {b} kv {kh}")
