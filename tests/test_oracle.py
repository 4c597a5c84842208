"""Pins of the fp64 oracle against facts fixed outside it (CPU only).

Each test checks the oracle against something it does not compute itself: hand-derived sets and
values under tests/golden/, closed forms, a textbook library routine (PyTorch SDPA) in the cases
where the method reduces to it, invariants of softmax attention, and a second, independently
written formulation (C brute-force predicate scan versus numpy range construction).
"""
import math
import os

import numpy as np
import pytest
import torch

from oracle.reference import (OracleLib, Problem, attention, attention_row, bf16_round, build_pool,
                              pages_bytes, rope_cos_sin, rope_rotate_bf16, rope_rotate_f64,
                              stored_logical_pages, visible_keys)

GOLD = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rows(name):
    out = []
    with open(os.path.join(GOLD, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                cols = [c.strip() for c in line.split("|")]
                out.append(cols[0].split() + cols[1:])
    return out


def _ranges(txt):
    if txt == "-":
        return []
    s = []
    for part in txt.split(","):
        if "-" in part:
            a, b = part.split("-")
            s.extend(range(int(a), int(b) + 1))
        else:
            s.append(int(part))
    return s


@pytest.fixture(scope="module")
def lib():
    return OracleLib()


def _problem(rng, seqs, Hq, Hkv, D, classes, scale_q=1.0):
    """Random bf16-valued problem. seqs: [(L, Lq)]; classes: [B][Hkv] of (is_global, S, W)."""
    cu_k = np.concatenate([[0], np.cumsum([s[0] for s in seqs])]).astype(np.int32)
    cu_q = np.concatenate([[0], np.cumsum([s[1] for s in seqs])]).astype(np.int32)
    q = bf16_round(rng.standard_normal((cu_q[-1], Hq, D)).astype(np.float32) * scale_q)
    k = bf16_round(rng.standard_normal((cu_k[-1], Hkv, D)).astype(np.float32))
    v = bf16_round(rng.standard_normal((cu_k[-1], Hkv, D)).astype(np.float32))
    c = np.asarray(classes, dtype=np.int32)
    return Problem(q, k, v, cu_q, cu_k, c[..., 0].copy(), c[..., 1].copy(), c[..., 2].copy())


# ------------------------------------------------------------------------------------------ sets

def test_visible_sets_match_hand_derived():
    for cls, S, W, i, want, n in _rows("visible_sets.txt"):
        g = cls == "global"
        got = visible_keys(g, int(S), int(W), int(i))
        assert list(got) == _ranges(want), (cls, S, W, i)
        assert len(got) == int(n)


def test_c_bruteforce_set_sizes_match_hand_derived(lib):
    """The C oracle enumerates V(i) by scanning every key; its |V(i)| must match the golden sizes."""
    rng = np.random.default_rng(0)
    for cls, S, W, i, want, n in _rows("visible_sets.txt"):
        i = int(i)
        pb = _problem(rng, [(i + 1, 1)], 1, 1, 4, [[(int(cls == "global"), int(S), int(W))]])
        p, cnt = lib.probs(pb, 0, 0, 1.0)
        assert cnt == int(n)
        assert sorted(np.nonzero(p)[0].tolist()) == _ranges(want)


def test_uniform_attention_recovers_the_set():
    """Q = 0 makes every visible logit 0: O is the mean of the visible V rows, LSE = ln |V(i)|.
    With one-hot V rows, O's support is exactly V(i) (closed form)."""
    for cls, S, W, i, want, n in _rows("visible_sets.txt"):
        i = int(i)
        if i >= 80:
            continue
        L, D = i + 1, 80
        v = np.zeros((L, 1, D), np.float32)
        v[np.arange(L), 0, np.arange(L)] = 1.0
        pb = Problem(np.zeros((1, 1, D), np.float32), np.ones((L, 1, D), np.float32), v,
                     np.array([0, 1], np.int32), np.array([0, L], np.int32),
                     np.array([[int(cls == "global")]]), np.array([[int(S)]]), np.array([[int(W)]]))
        o, lse, _, _ = attention_row(pb, 0, 0, 0.0)
        assert sorted(np.nonzero(o)[0].tolist()) == _ranges(want)
        np.testing.assert_allclose(o[np.nonzero(o)[0]], 1.0 / int(n), rtol=0, atol=1e-15)
        assert abs(lse - math.log(int(n))) < 1e-13


def test_uniform_golden_value(lib):
    (_, p, lse), = [r for r in _rows("closed_forms.txt") if r[0] == "uniform_n68"]
    pb = _problem(np.random.default_rng(1), [(256, 64)], 2, 1, 8, [[(0, 4, 64)]])
    pb.q[:] = 0.0
    o, l = lib.attention(pb, 1.0, items=[(8, 1)])           # row 8 -> position 200, 68 visible keys
    assert abs(l[0] - float(lse)) < 1e-13
    pr, n = lib.probs(pb, 8, 1, 1.0)
    assert n == 68 and np.allclose(pr[pr > 0], float(p), atol=1e-15)


def test_two_key_closed_form(lib):
    (_, o_want, lse_want), = [r for r in _rows("closed_forms.txt") if r[0] == "two_key"]
    o_want = np.array([float(x) for x in o_want.split()])
    q = np.array([[[np.float32(math.log(3.0)), 0.0]]], np.float32)
    k = np.array([[[0.0, 0.0]], [[1.0, 0.0]]], np.float32)
    v = np.array([[[1.0, 0.0]], [[0.0, 1.0]]], np.float32)
    pb = Problem(q, k, v, np.array([0, 1], np.int32), np.array([0, 2], np.int32),
                 np.array([[1]]), np.array([[0]]), np.array([[0]]))
    o1, l1, _, _ = attention_row(pb, 0, 0, 1.0)
    o2, l2 = lib.attention(pb, 1.0)
    for o, l in ((o1, l1), (o2[0], l2[0])):
        np.testing.assert_allclose(o, o_want, atol=1e-7)
        assert abs(l - float(lse_want)) < 1e-7


# ------------------------------------------------------------------ reductions to textbook cases

def _sdpa_tail(pb: Problem, b: int, scale: float, rng):
    """Causal SDPA (fp64) over the whole sequence, then its last Lq rows: the global-head case."""
    L = int(pb.cu_k[b + 1] - pb.cu_k[b])
    Lq = int(pb.cu_q[b + 1] - pb.cu_q[b])
    G = pb.Hq // pb.Hkv
    qf = rng.standard_normal((L, pb.Hq, pb.D))
    qf[L - Lq:] = pb.q[pb.cu_q[b]:pb.cu_q[b + 1]]
    kk = torch.from_numpy(pb.k[pb.cu_k[b]:pb.cu_k[b + 1]].astype(np.float64)).repeat_interleave(G, dim=1)
    vv = torch.from_numpy(pb.v[pb.cu_k[b]:pb.cu_k[b + 1]].astype(np.float64)).repeat_interleave(G, dim=1)
    out = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(qf).transpose(0, 1)[None], kk.transpose(0, 1)[None], vv.transpose(0, 1)[None],
        is_causal=True, scale=scale)
    return out[0].transpose(0, 1)[L - Lq:].numpy()                      # [Lq, Hq, D]


@pytest.mark.parametrize("G", [1, 2, 4])
def test_global_heads_equal_causal_sdpa(lib, G):
    rng = np.random.default_rng(10 + G)
    Hkv, D = 2, 16
    seqs = [(37, 11), (5, 5), (64, 1)]
    pb = _problem(rng, seqs, Hkv * G, Hkv, D, [[(1, 0, 0)] * Hkv] * len(seqs))
    scale = 1.0 / math.sqrt(D)
    o_c, _ = lib.attention(pb, scale)
    o_np, _ = attention(pb, scale)
    o_c = o_c.reshape(-1, pb.Hq, D)
    o_np = o_np.reshape(-1, pb.Hq, D)
    for b in range(len(seqs)):
        ref = _sdpa_tail(pb, b, scale, rng)
        sl = slice(pb.cu_q[b], pb.cu_q[b + 1])
        np.testing.assert_allclose(o_c[sl], ref, atol=1e-12, rtol=0)
        np.testing.assert_allclose(o_np[sl], ref, atol=1e-12, rtol=0)


def test_wide_window_local_equals_global(lib):
    """A local head whose window covers the whole context sees exactly what a global head sees."""
    rng = np.random.default_rng(3)
    seqs = [(50, 50), (33, 7)]
    loc = _problem(rng, seqs, 4, 2, 16, [[(0, 5, 50), (0, 0, 1000)], [(0, 40, 33), (0, 2, 64)]])
    glob = Problem(loc.q, loc.k, loc.v, loc.cu_q, loc.cu_k, np.ones_like(loc.is_global), loc.sink, loc.window)
    o1, l1 = lib.attention(loc, 0.25)
    o2, l2 = lib.attention(glob, 0.25)
    np.testing.assert_allclose(o1, o2, atol=1e-14, rtol=0)
    np.testing.assert_allclose(l1, l2, atol=1e-14, rtol=0)


def test_single_query_global_is_one_softmax_row(lib):
    rng = np.random.default_rng(4)
    pb = _problem(rng, [(40, 1)], 1, 1, 8, [[(1, 0, 0)]])
    s = 0.5 * (pb.k[:, 0, :].astype(np.float64) @ pb.q[0, 0].astype(np.float64))
    p = np.exp(s - s.max())
    p /= p.sum()
    o, l = lib.attention(pb, 0.5)
    np.testing.assert_allclose(o[0], p @ pb.v[:, 0, :].astype(np.float64), atol=1e-13)
    assert abs(l[0] - (s.max() + math.log(np.exp(s - s.max()).sum()))) < 1e-13


# ------------------------------------------------------------------------- two formulations agree

EDGE_SEQS = [
    ([(256, 64)], 4, 2, 64, [[(1, 0, 0), (0, 4, 64)]]),                       # the tiny layer
    ([(70, 70), (9, 1), (130, 3)], 8, 1, 16, [[(0, 3, 10)], [(0, 0, 1)], [(1, 0, 0)]]),
    ([(40, 40)], 8, 8, 8, [[(0, 50, 3), (0, 0, 40), (1, 0, 0), (0, 1, 1), (0, 39, 2), (0, 7, 7), (1, 0, 0), (0, 4, 64)]]),
    ([(1, 1), (2, 2)], 2, 2, 4, [[(0, 1, 1), (1, 0, 0)], [(0, 0, 1), (0, 5, 1)]]),
]


@pytest.mark.parametrize("case", range(len(EDGE_SEQS)))
def test_bruteforce_c_matches_range_numpy(lib, case):
    seqs, Hq, Hkv, D, classes = EDGE_SEQS[case]
    pb = _problem(np.random.default_rng(100 + case), seqs, Hq, Hkv, D, classes)
    o1, l1 = lib.attention(pb, 1.0 / math.sqrt(D))
    o2, l2 = attention(pb, 1.0 / math.sqrt(D))
    np.testing.assert_allclose(o1, o2, atol=1e-12, rtol=0)
    np.testing.assert_allclose(l1, l2, atol=1e-12, rtol=0)


# ------------------------------------------------------------------------------------ invariants

def test_rows_sum_to_one_and_lse_bounds(lib):
    pb = _problem(np.random.default_rng(5), [(300, 40)], 4, 2, 32, [[(1, 0, 0), (0, 8, 50)]], scale_q=3.0)
    scale = 1.0 / math.sqrt(32)
    o, lse = lib.attention(pb, scale)
    t = 0
    for r in range(pb.q.shape[0]):
        for h in range(pb.Hq):
            p, n = lib.probs(pb, r, h, scale)
            assert abs(p.sum() - 1.0) < 1e-12
            _, i = pb.row_seq_pos(r)
            vis = np.nonzero(p)[0]
            s = scale * (pb.k[vis, h // 2, :].astype(np.float64) @ pb.q[r, h].astype(np.float64))
            assert s.max() <= lse[t] + 1e-12 and lse[t] <= s.max() + math.log(n) + 1e-12
            vv = pb.v[vis, h // 2, :]
            assert np.all(o[t] >= vv.min(0) - 1e-12) and np.all(o[t] <= vv.max(0) + 1e-12)
            t += 1


def test_logit_shift_invariance(lib):
    pb = _problem(np.random.default_rng(6), [(120, 30)], 2, 1, 16, [[(0, 4, 20)]])
    o0, l0 = lib.attention(pb, 0.25)
    o1, l1 = lib.attention(pb, 0.25, shift=7.25)
    np.testing.assert_allclose(o1, o0, atol=1e-13)
    np.testing.assert_allclose(l1, l0 + 7.25, atol=1e-12)


def test_planted_visibility_mistakes_are_caught():
    """Each plausible slip in the visibility rule fails the hand-derived golden sets."""
    mutants = {
        "window_off_by_one": lambda g, S, W, i: np.arange(0, i + 1) if g else np.union1d(np.arange(min(S, i + 1)), np.arange(max(i - W, 0), i + 1)),
        "sink_inclusive": lambda g, S, W, i: np.arange(0, i + 1) if g else np.union1d(np.arange(min(S + 1, i + 1)), np.arange(max(i - W + 1, 0), i + 1)),
        "sink_not_causal": lambda g, S, W, i: np.arange(0, i + 1) if g else np.union1d(np.arange(S), np.arange(max(i - W + 1, 0), i + 1)),
        "no_self": lambda g, S, W, i: np.arange(0, i) if g else np.union1d(np.arange(min(S, i)), np.arange(max(i - W + 1, 0), i)),
    }
    gold = _rows("visible_sets.txt")
    for name, f in mutants.items():
        bad = sum(list(f(c == "global", int(S), int(W), int(i))) != _ranges(w) for c, S, W, i, w, _ in gold)
        assert bad > 0, name


# ------------------------------------------------------------------------- storage and footprint

def test_stored_pages_match_hand_derived():
    for cls, L, Lq, S, W, P, want, n in _rows("stored_pages.txt"):
        got = stored_logical_pages(int(L), int(Lq), cls == "global", int(S), int(W), int(P))
        assert got == _ranges(want), (cls, L, Lq, S, W, P)
        assert len(got) == int(n)


def test_pages_bytes_tiny_layer():
    """Tiny layer: 16 global + 9 local pages of 16 x 64 bf16, K and V; dense keeps 2 x 16 pages."""
    cu_k = np.array([0, 256]); cu_q = np.array([0, 64])
    stored, dense, per = pages_bytes(cu_k, cu_q, np.array([[1, 0]]), np.array([[0, 4]]), np.array([[0, 64]]), 16, 64)
    assert per.tolist() == [[16, 9]]
    assert stored == 25 * 16 * 64 * 2 * 2 and dense == 32 * 16 * 64 * 2 * 2


def test_build_pool_hand_example():
    """L=70, Lq=4, local S=4 W=2, P=16: the first query (66) reaches back to token 65, so the stored
    logical pages are {0, 4}; page 4 holds rows 64..69 then zeros."""
    L, D = 70, 4
    k = np.arange(L * D, dtype=np.float32).reshape(L, 1, D)
    v = -k
    assert stored_logical_pages(L, 4, False, 4, 2, 16) == [0, 4]
    kp, vp = build_pool(k, v, np.array([0, L]), np.array([0, 4]), np.array([[0]]), np.array([[4]]), np.array([[2]]),
                        16, np.array([7, 2]), np.array([0, 2]), 9)
    np.testing.assert_array_equal(kp[7], k[0:16, 0])
    np.testing.assert_array_equal(kp[2, :6], k[64:70, 0])
    np.testing.assert_array_equal(kp[2, 6:], 0)
    np.testing.assert_array_equal(vp[2, :6], v[64:70, 0])
    assert np.isnan(kp[0]).all() and np.isnan(vp[8]).all()


# ---------------------------------------------------------------------------------------- RoPE

def test_rope_table_closed_forms():
    t = rope_cos_sin(1e6, [0, 1], 8)
    assert np.all(t[0, :, 0] == 1.0) and np.all(t[0, :, 1] == 0.0)
    assert t[1, 0, 0] == np.float32(math.cos(1.0)) and t[1, 0, 1] == np.float32(math.sin(1.0))
    assert t[1, 1, 0] == np.float32(math.cos(1e6 ** (-2 / 8)))


def test_rope_zero_delta_is_identity_bitwise():
    x = bf16_round(np.random.default_rng(7).standard_normal((5, 64)).astype(np.float32))
    np.testing.assert_array_equal(rope_rotate_bf16(x, rope_cos_sin(1e6, [0], 64)[0]), x)


def test_rope_rotation_algebra_fp64():
    rng = np.random.default_rng(8)
    D = 64
    inv = 1e6 ** (-2.0 * np.arange(D // 2) / D)
    x = rng.standard_normal((3, D))
    # back and forth
    np.testing.assert_allclose(rope_rotate_f64(rope_rotate_f64(x, 123 * inv), -123 * inv), x, atol=1e-12)
    # composition
    np.testing.assert_allclose(rope_rotate_f64(rope_rotate_f64(x, 100 * inv), 23 * inv), rope_rotate_f64(x, 123 * inv), atol=1e-12)
    # the re-alignment itself: a key rotated at position p, then by delta, equals the key at p + delta
    p, delta = 517, 3001
    np.testing.assert_allclose(rope_rotate_f64(rope_rotate_f64(x, p * inv), delta * inv), rope_rotate_f64(x, (p + delta) * inv), atol=1e-10)


def test_rope_fp32_rule_within_bf16_rounding_of_exact():
    rng = np.random.default_rng(9)
    D = 128
    x = bf16_round(rng.standard_normal((50, D)).astype(np.float32))
    deltas = [0, 1, 77, 4095]
    tab = rope_cos_sin(1e6, deltas, D)
    inv = 1e6 ** (-2.0 * np.arange(D // 2) / D)
    for b, dlt in enumerate(deltas):
        got = rope_rotate_bf16(x, tab[b]).astype(np.float64)
        ref = rope_rotate_f64(x.astype(np.float64), dlt * inv)
        # bf16 keeps 8 significant bits: half an ulp is 2^-8 relative, plus fp32 table/product rounding
        assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-6)
