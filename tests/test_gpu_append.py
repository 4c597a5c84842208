"""segpaged_attn_prefill_append (fused append-and-attend) on the GPU against the fp64 oracle.

The pool is built with unrelated values in every query row; one fused launch must write the query rows'
new keys and values into their pages and attend over the pool's earlier rows plus the new rows. Checked:
O / LSE on every row against the oracle on the true K/V (small and split shapes), sampled rows at full size,
and the whole pool afterwards bit-exact against the oracle's build of the true K/V.
"""
import numpy as np
import pytest
import torch

from head_sparse_paged_b200 import synth
from head_sparse_paged_b200.runner import Runner
from oracle import reference as orc

from gpu_common import compare, full_problem, head_problem, sample_rows
from test_gpu_prefill import SMALL

pytestmark = pytest.mark.gpu

_LIB = None


def lib():
    global _LIB
    if _LIB is None:
        _LIB = orc.OracleLib()
    return _LIB


def _run(w, **kw):
    kw.setdefault("keep_dense", True)
    r = Runner(w, append=True, **kw)
    for li in r.layers:
        r.prefill(li)
    torch.cuda.synchronize()
    r.check_status()
    return r


def _check_pool(w, r, li):
    st = r.state[li]
    k, v = r.dense[li]
    c = w.classes[li]
    kp, vp = orc.build_pool(k.float().cpu().numpy(), v.float().cpu().numpy(), w.cu_k(), w.cu_q(), c[..., 0], c[..., 1],
                            c[..., 2], w.page_size, st.table, st.offs, r.num_pages)
    used = ~np.isnan(kp[:, 0, 0])
    np.testing.assert_array_equal(r.k_pool.float().cpu().numpy()[used], kp[used])
    np.testing.assert_array_equal(r.v_pool.float().cpu().numpy()[used], vp[used])


CASES = {name: SMALL[name] for name in ("tiny", "varlen-p16-g4", "mha-d64-p128", "g16-p64", "g8-p32")}
CASES["q0-mid-page"] = lambda: synth.custom("q0-mid-page", [(1000, 333), (77, 77), (600, 1)], 8, 2, 128, 64,
                                            [[(1, 0, 0), (0, 16, 100)], [(0, 3, 5), (1, 0, 0)], [(0, 700, 9), (0, 0, 600)]],
                                            seed=71)
# a decode-like batch: every unit a half unit, split chunks with odd tile counts
CASES["llama-decode8x16"] = lambda: synth.llama_70b_decode(8, 16)


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("split", [0, None])
def test_append_matches_oracle_every_row_and_writes_the_pool(name, split):
    w = CASES[name]()
    r = _run(w, split_ctas=(1000 if split is None else 0))
    st = r.state[0]
    k, v = r.dense[0]
    pb = full_problem(w, 0, st.q.float().cpu().numpy(), k.float().cpu().numpy(), v.float().cpu().numpy())
    items = np.array([(row, h) for row in range(w.total_q) for h in range(w.num_q_heads)], np.int64)
    o_ref, lse_ref = lib().attention(pb, r.scale, items)
    compare(st.o.float().cpu().numpy().reshape(-1, w.head_dim), st.lse.cpu().numpy().T.reshape(-1), o_ref, lse_ref,
            f"{name} split={split}")
    _check_pool(w, r, 0)


@pytest.mark.parametrize("name", ["qwen3-32b", "llama-3.3-70b"])
def test_append_full_size_sampled_and_pool(name):
    w = synth.get(name)
    r = _run(w)
    st = r.state[0]
    k, v = r.dense[0]
    rng = np.random.default_rng(8)
    G = w.group
    for b in range(w.num_seqs):
        for kh in sorted(rng.choice(w.num_kv_heads, 3, replace=False)):
            pb = head_problem(w, 0, b, int(kh), st.q, k, v)
            rows = sample_rows(w.q_lens[b], 128 // G, rng, extra=2)
            items = np.array([(row, h) for row in rows for h in range(G)], np.int64)
            o_ref, lse_ref = lib().attention(pb, r.scale, items)
            gr = torch.tensor([int(w.cu_q()[b]) + row for row in rows for _ in range(G)], device=st.o.device)
            gh = torch.tensor([int(kh) * G + h for _ in rows for h in range(G)], device=st.o.device)
            compare(st.o[gr, gh].float().cpu().numpy(), st.lse[gh, gr].cpu().numpy(), o_ref, lse_ref,
                    f"{name} seq {b} kv {kh}")
    # the query rows' pages hold the new keys and values
    ck, ql = w.cu_k(), w.q_lens
    for b in range(w.num_seqs):
        L = w.ctx_lens[b]
        for kh in range(w.num_kv_heads):
            g, S, W = (int(x) for x in w.classes[0, b, kh])
            stored = orc.stored_logical_pages(L, ql[b], bool(g), S, W, w.page_size)
            base = int(st.offs[b * w.num_kv_heads + kh])
            for pos in (L - ql[b], L - 1, L - ql[b] + ql[b] // 2):
                t = stored.index(pos // w.page_size)
                pid = int(st.table[base + t])
                row = pos % w.page_size
                assert torch.equal(r.k_pool[pid, row], k[int(ck[b]) + pos, kh])
                assert torch.equal(r.v_pool[pid, row], v[int(ck[b]) + pos, kh])
