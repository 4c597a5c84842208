"""Pins of the oracle's token-mass score and top-k selection (CPU only).

The mass a token receives is checked against a second, independent formulation (C brute-force
predicate scan versus numpy index ranges), against closed forms for uniform attention (all logits
equal, so each row spreads its probability evenly over its visible set), and against the softmax
invariant that every query row hands out exactly one unit of probability per head. The selection is
checked against hand-derived cases in tests/golden/topk_select.txt.
"""
import os

import numpy as np
import pytest

from oracle.reference import OracleLib, Problem, bf16_round, select_topk, token_mass

GOLD = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


@pytest.fixture(scope="module")
def lib():
    return OracleLib()


def _problem(rng, seqs, Hq, Hkv, D, classes, zero_q=False):
    cu_k = np.concatenate([[0], np.cumsum([s[0] for s in seqs])]).astype(np.int32)
    cu_q = np.concatenate([[0], np.cumsum([s[1] for s in seqs])]).astype(np.int32)
    q = bf16_round(rng.standard_normal((cu_q[-1], Hq, D)).astype(np.float32))
    if zero_q:
        q[:] = 0.0
    k = bf16_round(rng.standard_normal((cu_k[-1], Hkv, D)).astype(np.float32))
    v = bf16_round(rng.standard_normal((cu_k[-1], Hkv, D)).astype(np.float32))
    c = np.asarray(classes, dtype=np.int32)
    return Problem(q, k, v, cu_q, cu_k, c[..., 0].copy(), c[..., 1].copy(), c[..., 2].copy())


def test_mass_c_bruteforce_matches_numpy_ranges(lib):
    rng = np.random.default_rng(41)
    pb = _problem(rng, [(70, 40), (33, 33), (9, 0), (50, 7)], 4, 2, 16,
                  [[(1, 0, 0), (0, 3, 8)], [(0, 0, 5), (0, 40, 2)], [(1, 0, 0), (1, 0, 0)], [(0, 2, 100), (0, 60, 1)]])
    a = lib.token_mass(pb, 0.25)
    b = token_mass(pb, 0.25)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)


def test_mass_full_range_sums_to_rows_times_heads(lib):
    """With the query range = the whole sequence, every key is scored, so the masses add up to the
    probability every (row, head) hands out: exactly one each."""
    rng = np.random.default_rng(42)
    pb = _problem(rng, [(57, 57), (20, 20)], 8, 2, 16, [[(1, 0, 0), (0, 4, 9)], [(0, 0, 1), (0, 30, 3)]])
    m = lib.token_mass(pb, 0.3)
    for b in range(2):
        lo, hi = pb.cu_q[b], pb.cu_q[b + 1]
        assert abs(m[lo:hi].sum() - 8 * (hi - lo)) < 1e-9


def test_mass_partial_range_is_bounded(lib):
    rng = np.random.default_rng(43)
    pb = _problem(rng, [(90, 30)], 4, 1, 16, [[(1, 0, 0)]])
    m = lib.token_mass(pb, 0.3)
    assert (m > 0).all()
    assert m.sum() < 4 * 30
    # the last token is seen only by the last row: its mass is at most one per head
    assert m[-1] <= 4 + 1e-12


def test_mass_uniform_attention_global_closed_form(lib):
    """Q = 0: every visible logit is 0, so row i gives 1/(i+1) to each key of [0, i]. Token j of a
    global head with the whole sequence queried receives sum_{i=j}^{L-1} 1/(i+1) per head."""
    L, H = 40, 3
    pb = _problem(np.random.default_rng(44), [(L, L)], H, 1, 8, [[(1, 0, 0)]], zero_q=True)
    m = lib.token_mass(pb, 1.0)
    want = np.array([H * sum(1.0 / (i + 1) for i in range(j, L)) for j in range(L)])
    np.testing.assert_allclose(m, want, rtol=1e-12)
    np.testing.assert_allclose(token_mass(pb, 1.0), want, rtol=1e-12)


def test_mass_uniform_attention_window_closed_form(lib):
    """Q = 0, local head with no sink and window W, tail query range: row i spreads over
    [max(i-W+1, 0), i], so token j receives sum over i in [j, min(j+W-1, L-1)] of 1/min(W, i+1)."""
    L, Lq, W, H = 50, 23, 6, 2
    pb = _problem(np.random.default_rng(45), [(L, Lq)], H, 1, 8, [[(0, 0, W)]], zero_q=True)
    m = lib.token_mass(pb, 1.0)
    q0 = L - Lq
    want = np.array([H * sum(1.0 / min(W, i + 1) for i in range(j, min(j + W, L))) for j in range(q0, L)])
    np.testing.assert_allclose(m, want, rtol=1e-12)
    np.testing.assert_allclose(token_mass(pb, 1.0), want, rtol=1e-12)


def test_mass_uniform_attention_sink_closed_form(lib):
    """Q = 0, local head with sink S and window W, whole sequence queried: |V(i)| is
    min(S, i+1) + the window keys past the sink; a token past the sink is seen by rows within W."""
    L, S, W = 30, 4, 5
    pb = _problem(np.random.default_rng(46), [(L, L)], 1, 1, 8, [[(0, S, W)]], zero_q=True)
    m = lib.token_mass(pb, 1.0)

    def nvis(i):
        lo = max(i - W + 1, 0)
        return min(S, i + 1) + (i - max(lo, S) + 1 if i >= max(lo, S) else 0)

    want = []
    for j in range(L):
        rows = range(j, L) if j < S else range(j, min(j + W, L))
        want.append(sum(1.0 / nvis(i) for i in rows))
    np.testing.assert_allclose(m, np.array(want), rtol=1e-12)


def _golden():
    out = []
    with open(os.path.join(GOLD, "topk_select.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                cols = [c.strip() for c in line.split("|")]
                want = [] if cols[3] == "-" else [int(x) for x in cols[3].split()]
                out.append(([float(x) for x in cols[0].split()], [int(x) for x in cols[1].split()],
                            [int(x) for x in cols[2].split()], want))
    return out


@pytest.mark.parametrize("case", range(len(_golden())))
def test_select_topk_matches_hand_derived(case):
    mass, cu, k, want = _golden()[case]
    assert select_topk(np.array(mass), np.array(cu), np.array(k)).tolist() == want
