"""Pins of the oracle's bf16 rounding and of its fp32 RoPE rotation rule, bit for bit (CPU).

The build's RoPE re-alignment is required to be bit-exact, so the oracle's rounding rule (``bf16_round``) and the
order of its rounded operations (``rope_rotate_bf16``) must be fixed by something other than the oracle itself:
  * hand-derived float32 -> bf16 words (tests/golden/bf16_round.txt): ties with even and odd upper halves, one ulp
    either side of a tie, carries into the exponent, overflow to infinity, subnormals, signed zeros;
  * the same words from PyTorch's CPU float32 -> bfloat16 conversion (a textbook round-to-nearest-even), on the
    golden words and on random finite words;
  * two hand-derived RoPE vectors (tests/golden/rope_rotate_bf16.txt) whose words change under a fused
    multiply-add, a ties-away rounding, interleaved pairs or the other rotation sign.
Each plausible slip is planted here, on the CPU, and must fail one of the golden words.
Source of the rule: rotating offline keys to their actual position ("RedKnot – 小红书研发并开源的长上下文大模型推理引擎",
shshi.cn, 技术原理 2 "位置无关缓存复用", item "RoPE位置对齐").
"""
import os

import numpy as np
import torch

from oracle import reference as orc

GOLD = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rows(name):
    out = []
    with open(os.path.join(GOLD, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                out.append([part.strip() for part in line.split("|")])
    return out


def _bf16_cases():
    rows = _rows("bf16_round.txt")
    f32 = np.array([int(r[0], 16) for r in rows], np.uint32)
    bf = np.array([int(r[1], 16) for r in rows], np.uint32)
    return f32, bf


def _bits_after(fn, words: np.ndarray) -> np.ndarray:
    """Upper 16 bits of fn(float32 values of `words`)."""
    with np.errstate(over="ignore", invalid="ignore"):
        out = fn(words.view(np.float32))
    u = np.ascontiguousarray(out, dtype=np.float32).view(np.uint32)
    assert np.all((u & 0xFFFF) == 0), "bf16 values must have a zero lower half"
    return u >> 16


def test_bf16_round_golden_words():
    f32, bf = _bf16_cases()
    got = _bits_after(orc.bf16_round, f32)
    bad = [(hex(a), hex(b), hex(c)) for a, b, c in zip(f32, bf, got) if b != c]
    assert not bad, bad


def test_bf16_golden_words_match_torch_conversion():
    """The hand-derived words agree with PyTorch's CPU float32 -> bfloat16 conversion."""
    f32, bf = _bf16_cases()
    t = torch.from_numpy(f32.view(np.float32).copy()).to(torch.bfloat16).view(torch.int16).numpy()
    assert np.array_equal(t.astype(np.uint16).astype(np.uint32), bf)


def test_bf16_round_matches_torch_on_random_words():
    rng = np.random.default_rng(7)
    w = rng.integers(0, 1 << 32, size=200000, dtype=np.uint64).astype(np.uint32)
    w = w[np.isfinite(w.view(np.float32))]
    ties = (w & np.uint32(0xFFFF0000)) | np.uint32(0x8000)       # every tie, both parities
    for words in (w, ties[np.isfinite(ties.view(np.float32))]):
        ours = _bits_after(orc.bf16_round, words)
        ref = torch.from_numpy(words.view(np.float32).copy()).to(torch.bfloat16).view(torch.int16).numpy()
        assert np.array_equal(ours, ref.astype(np.uint16).astype(np.uint32))


def _ties_away(x):
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return (((u + 0x8000) >> 16).astype(np.uint32) << 16).view(np.float32)


def _truncate(x):
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return (u & np.uint32(0xFFFF0000)).view(np.float32)


def _ties_odd(x):
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + (1 - ((u >> 16) & 1))) >> 16
    return (u.astype(np.uint32) << 16).view(np.float32)


def _no_overflow(x):
    """Saturates at the largest finite bf16 instead of rounding to infinity."""
    y = orc.bf16_round(x)
    big = np.float32(np.uint32(0x7F7F0000).view(np.float32))
    return np.where(np.isinf(y) & np.isfinite(x), np.copysign(big, x), y).astype(np.float32)


def test_planted_rounding_mistakes_fail_the_golden_words():
    f32, bf = _bf16_cases()
    for mutant in (_ties_away, _truncate, _ties_odd, _no_overflow):
        with np.errstate(over="ignore", invalid="ignore"):
            got = np.ascontiguousarray(mutant(f32.view(np.float32)), dtype=np.float32).view(np.uint32) >> 16
        assert not np.array_equal(got, bf), mutant.__name__


def _rope_cases():
    out = []
    for name, x, tab, y in _rows("rope_rotate_bf16.txt"):
        xw = np.array([int(v, 16) << 16 for v in x.split()], np.uint32).view(np.float32)
        tw = np.array([int(v, 16) for v in tab.split()], np.uint32).view(np.float32).reshape(-1, 2)
        yw = np.array([int(v, 16) for v in y.split()], np.uint32)
        out.append((name, xw, tw, yw))
    return out


def _words(y):
    u = np.ascontiguousarray(y, dtype=np.float32).view(np.uint32)
    assert np.all((u & 0xFFFF) == 0)
    return u >> 16


def test_rope_rotate_golden_vectors():
    for name, x, tab, y in _rope_cases():
        got = _words(orc.rope_rotate_bf16(x[None, :], tab)[0])
        assert np.array_equal(got, y), (name, [hex(v) for v in got], [hex(v) for v in y])


def _rope_fused(x, cs):
    """Planted mistake: the first product of each output fused with the sum (one rounding), as a compiler that
    contracts x1*c - (x2*s) into an FMA would evaluate it. float64 holds the float32 x bf16 product exactly and
    the sum with a float32 of nearby exponent exactly, so one float32 rounding follows."""
    D = x.shape[-1]
    x1, x2 = x[..., : D // 2].astype(np.float64), x[..., D // 2:].astype(np.float64)
    c, s = cs[:, 0].astype(np.float64), cs[:, 1].astype(np.float64)
    y1 = (x1 * c - (x2 * s).astype(np.float32)).astype(np.float32)
    y2 = (x2 * c + (x1 * s).astype(np.float32)).astype(np.float32)
    return orc.bf16_round(np.concatenate([y1, y2], axis=-1))


def _rope_interleaved(x, cs):
    y = np.empty_like(x, dtype=np.float32)
    a, b = x[..., 0::2].astype(np.float32), x[..., 1::2].astype(np.float32)
    c, s = cs[:, 0], cs[:, 1]
    y[..., 0::2] = np.float32(a * c) - np.float32(b * s)
    y[..., 1::2] = np.float32(b * c) + np.float32(a * s)
    return orc.bf16_round(y)


def _rope_other_sign(x, cs):
    return orc.rope_rotate_bf16(x, np.stack([cs[:, 0], -cs[:, 1]], axis=-1))


def _rope_ties_away(x, cs):
    D = x.shape[-1]
    x1, x2 = x[..., : D // 2].astype(np.float32), x[..., D // 2:].astype(np.float32)
    c, s = cs[:, 0], cs[:, 1]
    y = np.concatenate([np.float32(x1 * c) - np.float32(x2 * s), np.float32(x2 * c) + np.float32(x1 * s)], axis=-1)
    return _ties_away(y)


def test_planted_rope_mistakes_fail_the_golden_vectors():
    cases = _rope_cases()
    for mutant in (_rope_fused, _rope_interleaved, _rope_other_sign, _rope_ties_away):
        hit = any(not np.array_equal(_words(mutant(x[None, :], tab)[0]), y) for _, x, tab, y in cases)
        assert hit, mutant.__name__
