"""Pins of the oracle's gather-time (per-fragment) RoPE re-alignment (CPU only).

The fragment a token belongs to is checked against hand-derived cases (tests/golden/rope_fragments.txt);
the re-aligned keys are checked end to end against the closed form of rotary embedding: keys computed at
their original positions and re-aligned by delta = actual - original agree with keys computed at their
actual positions, in fp64, to bf16 rounding.
"""
import os

import numpy as np

from oracle.reference import (bf16_round, rope_cos_sin, rope_fragment_keys, rope_fragment_of, rope_rotate_bf16,
                              rope_rotate_f64)

GOLD = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_fragment_of_matches_hand_derived():
    n = 0
    with open(os.path.join(GOLD, "rope_fragments.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            starts_txt, want_txt = (c.strip() for c in line.split("|"))
            starts = [] if starts_txt == "-" else [int(x) for x in starts_txt.split()]
            want = [int(x) for x in want_txt.split()]
            assert [rope_fragment_of(starts, t) for t in range(len(want))] == want, starts
            n += 1
    assert n == 5


def test_fragment_keys_realign_to_actual_positions():
    """Two sequences; sequence 0 is three reused fragments whose keys were computed at offsets other than
    where they now sit, sequence 1 has an unrotated prefix before its only fragment."""
    rng = np.random.default_rng(21)
    D, H, theta = 64, 2, 1e6
    inv = theta ** (-2.0 * np.arange(D // 2) / D)
    L = [40, 25]
    cu_k = np.array([0, 40, 65], np.int32)
    # (start, original position of the fragment's first token)
    frags = [[(0, 1000), (13, 7), (30, 30)], [(10, 500)]]
    x = rng.standard_normal((65, H, D))                     # position-free content of every key
    offline = np.zeros((65, H, D))                          # keys as computed offline (original positions)
    actual = np.zeros((65, H, D))                           # keys computed where the tokens now sit
    starts, deltas = [], []
    for b in range(2):
        fl = frags[b]
        for j in range(L[b]):
            f = max([i for i, (s0, _) in enumerate(fl) if s0 <= j], default=-1)
            orig = j if f < 0 else fl[f][1] + (j - fl[f][0])
            row = cu_k[b] + j
            offline[row] = rope_rotate_f64(x[row], orig * inv)
            actual[row] = rope_rotate_f64(x[row], j * inv)
        starts += [s0 for s0, _ in fl]
        deltas += [s0 - o for s0, o in fl]
    offs = np.array([0, 3, 4], np.int32)
    cs = rope_cos_sin(theta, deltas, D)
    k = bf16_round(offline.astype(np.float32))
    got = rope_fragment_keys(k, cu_k, offs, np.array(starts, np.int32), cs).astype(np.float64)
    # each key: bf16 input rounding, fp32 table and products, bf16 output rounding
    err = np.abs(got - actual)
    assert np.all(err <= 2.0 ** -7 * np.abs(actual) + 2.0 ** -7 * np.abs(offline).max(axis=-1, keepdims=True))
    # tokens before the first fragment keep their keys bit for bit
    np.testing.assert_array_equal(got[40:50], k[40:50].astype(np.float64))


def test_fragment_keys_single_fragment_equals_whole_sequence_rotation():
    rng = np.random.default_rng(22)
    k = bf16_round(rng.standard_normal((30, 3, 128)).astype(np.float32))
    cs = rope_cos_sin(1e6, [4321], 128)
    got = rope_fragment_keys(k, np.array([0, 30], np.int32), np.array([0, 1], np.int32), np.array([0], np.int32), cs)
    np.testing.assert_array_equal(got, rope_rotate_bf16(k, cs[0]))
