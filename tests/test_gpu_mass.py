"""segpaged_token_mass and segpaged_select_topk on the GPU against the fp64 oracle.

Mass: every row of the small and mid-size shapes is compared with the oracle's token mass (C brute
force), relative tolerance MASS_RTOL. At full size (Qwen3-shaped layer, the 43-layer workload's mixed
layer) the last tokens of the query range, which only the last rows see, are computed by the oracle one
by one; every token is checked against the bounds that hold at any size. The selection is bit-exact
against the oracle's selection rule applied to the kernel's own masses (a float decides an integer:
both sides decide on the same fp32 values), and agrees with the selection on the oracle's masses
except between near-equal masses.
"""
import numpy as np
import pytest
import torch

from head_sparse_paged_b200 import synth
from head_sparse_paged_b200.runner import Runner
from oracle import reference as orc

from gpu_common import full_problem, oracle_dense
from test_gpu_prefill import SMALL, SPLIT

pytestmark = pytest.mark.gpu

# fp32 logits from bf16 operands, the prefill's fp32 LSE, ex2.approx and fp32 sums: relative error of a
# token's mass well under 1e-4 in practice; the bar leaves an order of magnitude.
MASS_RTOL = 2e-3
MASS_ATOL = 1e-5

_LIB = None


def lib():
    global _LIB
    if _LIB is None:
        _LIB = orc.OracleLib()
    return _LIB


def _run(w, **kw):
    kw.setdefault("keep_dense", True)
    r = Runner(w, mass=True, **kw)
    for li in r.layers:
        r.prefill(li)
        r.token_mass(li)
    torch.cuda.synchronize()
    r.check_status()
    return r


CASES = dict(SMALL)
CASES["split-short-q"] = SPLIT["split-short-q"][0]
CASES["qwen3-32b-lq64"] = lambda: synth.get("qwen3-32b-lq64")
CASES["llama-decode8x16"] = SPLIT["llama-decode8x16"][0]


@pytest.mark.parametrize("name", list(CASES))
def test_mass_matches_oracle_every_row(name):
    w = CASES[name]()
    r = _run(w)
    k, v = r.dense[0]
    qn, kn, vn = oracle_dense(w, r.state[0].q, k, v)
    ref = lib().token_mass(full_problem(w, 0, qn, kn, vn), r.scale)
    got = r.state[0].mass.cpu().numpy().astype(np.float64)
    err = np.abs(got - ref)
    assert np.all(np.isfinite(got))
    assert np.all(err <= MASS_RTOL * np.abs(ref) + MASS_ATOL), f"{name}: max rel {np.max(err / (ref + 1e-30)):.3e}"


def test_mass_is_bit_identical_under_page_permutation_and_repeat():
    w = SMALL["varlen-p16-g4"]()
    a = _run(w)
    b = _run(w, page_seed_offset=77)
    assert torch.equal(a.state[0].mass, b.state[0].mass)
    a.token_mass(0)
    torch.cuda.synchronize()
    assert torch.equal(a.state[0].mass, b.state[0].mass)


def _host_select(mass, cu, k):
    return orc.select_topk(mass, cu, k)


@pytest.mark.parametrize("name", ["varlen-p16-g4", "mistral-7b", "g16-p64"])
def test_select_topk_exact_on_kernel_masses(name):
    w = SMALL[name]()
    r = _run(w)
    m = r.state[0].mass.cpu().numpy()
    cu = w.cu_q()
    rng = np.random.default_rng(9)
    for trial in range(6):
        if trial == 0:
            k = np.zeros(w.num_seqs, np.int32)
        elif trial == 1:
            k = np.asarray(w.q_lens, np.int32) + 3
        elif trial == 2:
            k = -np.ones(w.num_seqs, np.int32)
        else:
            k = np.array([rng.integers(0, max(l, 1) + 1) for l in w.q_lens], np.int32)
        want = _host_select(m, cu, k)
        sel = torch.full((max(len(want), 1),), -7, dtype=torch.int32, device="cuda")
        r.select_topk(0, torch.from_numpy(k).cuda(), sel)
        torch.cuda.synchronize()
        got = sel.cpu().numpy()[: len(want)]
        assert got.tolist() == want.tolist(), (name, trial)


def test_select_topk_ties_and_large_sequences():
    """Many equal masses (the lower row wins) and sequences far longer than one block's threads."""
    rng = np.random.default_rng(10)
    lens = [5000, 1, 0, 20000, 1023, 1025]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    m = rng.integers(0, 7, size=int(cu[-1])).astype(np.float32) * 0.25   # heavy ties
    m[:100] = 3.0
    k = np.array([777, 1, 5, 12345, 1023, 1], np.int32)
    want = _host_select(m, cu, k)
    sel = torch.full((len(want),), -7, dtype=torch.int32, device="cuda")
    from head_sparse_paged_b200 import segpaged as sp
    sp.segpaged_select_topk(torch.from_numpy(m).cuda(), torch.from_numpy(cu).cuda(), torch.from_numpy(k).cuda(), sel)
    torch.cuda.synchronize()
    assert sel.cpu().numpy().tolist() == want.tolist()


def test_select_topk_agrees_with_oracle_masses_up_to_near_ties():
    w = SMALL["mistral-7b"]()
    r = _run(w)
    k, v = r.dense[0]
    qn, kn, vn = oracle_dense(w, r.state[0].q, k, v)
    ref = lib().token_mass(full_problem(w, 0, qn, kn, vn), r.scale)
    got = r.state[0].mass.cpu().numpy()
    cu = w.cu_q()
    kk = np.array([w.q_lens[0] // 8], np.int32)
    a = set(_host_select(got, cu, kk).tolist())
    b = set(_host_select(ref, cu, kk).tolist())
    thr = np.sort(ref)[::-1][kk[0] - 1]
    for row in a ^ b:
        assert abs(ref[row] - thr) <= 4 * MASS_RTOL * thr, (row, ref[row], thr)


FULL = {
    "qwen3-32b": lambda: (synth.qwen3_32b(), 0),
    "dsv4-flash-mixed-layer": lambda: (synth.dsv4_flash(layers=7), 3),
}


@pytest.mark.parametrize("name", list(FULL))
def test_mass_full_size_last_tokens_and_bounds(name):
    w, layer = FULL[name]()
    r = _run(w, layers=[layer])
    st = r.state[layer]
    got = st.mass.cpu().numpy().astype(np.float64)
    # bounds at any size: each row hands each token at most one unit per head, and at least its own
    # token's share is positive
    for b in range(w.num_seqs):
        lo, hi = int(w.cu_q()[b]), int(w.cu_q()[b + 1])
        L, Lq = w.ctx_lens[b], w.q_lens[b]
        seen_by = np.zeros(Lq)
        for kh in range(w.num_kv_heads):
            g, S, W = (int(x) for x in w.classes[layer, b, kh])
            j = np.arange(L - Lq, L)
            if g or S >= L:
                n = L - j
            else:
                n = np.where(j < S, L - j, np.minimum(L - j, W))
            seen_by += w.group * n
        assert np.all(got[lo:hi] > 0) and np.all(got[lo:hi] <= seen_by * (1 + 1e-5)), name
    # the last tokens of sequence 0 exactly: token j is seen only by rows at positions >= j
    k, v = r.dense[layer]
    qn, kn, vn = oracle_dense(w, st.q, k, v)
    pb = full_problem(w, layer, qn, kn, vn)
    Lq = w.q_lens[0]
    for t in (1, 2, 3):
        row = Lq - t
        want = 0.0
        for rr in range(row, Lq):
            for h in range(w.num_q_heads):
                p, _ = lib().probs(pb, rr, h, r.scale)
                want += p[w.ctx_lens[0] - Lq + row]
        assert abs(got[row] - want) <= MASS_RTOL * want + MASS_ATOL, (name, t, got[row], want)
