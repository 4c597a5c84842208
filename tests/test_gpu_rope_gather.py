"""segpaged_attn_prefill_rope (gather-time RoPE re-alignment per sequence fragment) on the GPU.

Bit-exact against the build-time re-alignment when each sequence is one fragment starting at 0 (the same
rotation and rounding, applied to the keys in shared memory instead of in the pool), for prefill and
token mass; with several fragments per sequence (starts inside pages and inside 128-key tiles, tokens
before the first fragment) every row against the oracle run on the oracle's own re-aligned keys.
"""
import numpy as np
import pytest
import torch

from head_sparse_paged_b200 import synth
from head_sparse_paged_b200.runner import Runner
from oracle import reference as orc

from gpu_common import compare, full_problem
from test_gpu_mass import MASS_ATOL, MASS_RTOL
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
    r = Runner(w, mass=True, **kw)
    r.prefill(0)
    r.token_mass(0)
    torch.cuda.synchronize()
    r.check_status()
    return r


@pytest.mark.parametrize("name", ["g2-p64", "mistral-7b"])
def test_one_fragment_per_sequence_equals_build_time_rope_bitwise(name):
    w = SMALL[name]()
    assert w.rope_theta is not None
    built = _run(w)
    tab = orc.rope_cos_sin(w.rope_theta, w.rope_deltas, w.head_dim)      # [B, D/2, 2]
    frags = (np.arange(w.num_seqs + 1, dtype=np.int32), np.zeros(w.num_seqs, np.int32), tab)
    gathered = _run(w, frags=frags)
    a, b = built.state[0], gathered.state[0]
    assert torch.equal(a.o, b.o) and torch.equal(a.lse, b.lse)
    assert torch.equal(a.mass, b.mass)


def _fragments(w, rng, per_seq):
    offs, starts, deltas = [0], [], []
    for b in range(w.num_seqs):
        L = w.ctx_lens[b]
        n = min(per_seq, max(L - 1, 0))
        st = sorted(set(int(x) for x in rng.integers(1, max(L, 2), size=n))) if n else []
        if b % 2 == 0 and L > 0:
            st = sorted(set([0] + st))                                   # some sequences start rotated
        starts += st
        deltas += [int(x) for x in rng.integers(-3000, 3000, size=len(st))]
        offs.append(len(starts))
    tab = orc.rope_cos_sin(1e4, deltas, w.head_dim) if deltas else np.zeros((1, w.head_dim // 2, 2), np.float32)
    return np.array(offs, np.int32), np.array(starts if starts else [0], np.int32), tab


CASES = ["tiny", "varlen-p16-g4", "mha-d64-p128", "g16-p64", "g8-p32"]


@pytest.mark.parametrize("name", CASES)
def test_many_fragments_match_oracle_every_row(name):
    w = SMALL[name]()
    w.rope_theta, w.rope_deltas = None, None
    rng = np.random.default_rng(sum(map(ord, name)))
    fo, fs, fc = _fragments(w, rng, per_seq=5)
    r = _run(w, frags=(fo, fs, fc))
    st = r.state[0]
    k, v = r.dense[0]
    qn = st.q.float().cpu().numpy()
    kn = orc.rope_fragment_keys(k.float().cpu().numpy(), w.cu_k(), fo, fs, fc)
    vn = v.float().cpu().numpy()
    pb = full_problem(w, 0, qn, kn, vn)
    items = np.array([(row, h) for row in range(w.total_q) for h in range(w.num_q_heads)], np.int64)
    o_ref, lse_ref = lib().attention(pb, r.scale, items)
    compare(st.o.float().cpu().numpy().reshape(-1, w.head_dim), st.lse.cpu().numpy().T.reshape(-1), o_ref, lse_ref,
            name)
    ref = lib().token_mass(pb, r.scale)
    got = st.mass.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - ref) <= MASS_RTOL * np.abs(ref) + MASS_ATOL), name


def test_fragments_with_split_plan_match_oracle():
    w = synth.custom("rope-split", [(3000, 9), (2000, 1), (700, 40)], 8, 2, 128, 64,
                     [[(1, 0, 0), (0, 64, 512)], [(0, 0, 300), (1, 0, 0)], [(1, 0, 0), (1, 0, 0)]], seed=61)
    rng = np.random.default_rng(62)
    fo, fs, fc = _fragments(w, rng, per_seq=7)
    r = _run(w, frags=(fo, fs, fc))
    st = r.state[0]
    assert st.info["num_groups"] > 0
    k, v = r.dense[0]
    kn = orc.rope_fragment_keys(k.float().cpu().numpy(), w.cu_k(), fo, fs, fc)
    pb = full_problem(w, 0, st.q.float().cpu().numpy(), kn, v.float().cpu().numpy())
    items = np.array([(row, h) for row in range(w.total_q) for h in range(w.num_q_heads)], np.int64)
    o_ref, lse_ref = lib().attention(pb, r.scale, items)
    compare(st.o.float().cpu().numpy().reshape(-1, w.head_dim), st.lse.cpu().numpy().T.reshape(-1), o_ref, lse_ref,
            "rope-split")


def test_fragments_on_a_decode_batch_match_oracle():
    """A decode-like batch (every unit a half unit, split chunks with odd tile counts) with several fragments
    per sequence."""
    w = synth.llama_70b_decode(8, 16)
    rng = np.random.default_rng(64)
    fo, fs, fc = _fragments(w, rng, per_seq=6)
    r = _run(w, frags=(fo, fs, fc))
    st = r.state[0]
    assert st.info["num_groups"] > 0 and st.info["num_half_units"] == st.info["num_units"]
    k, v = r.dense[0]
    kn = orc.rope_fragment_keys(k.float().cpu().numpy(), w.cu_k(), fo, fs, fc)
    pb = full_problem(w, 0, st.q.float().cpu().numpy(), kn, v.float().cpu().numpy())
    items = np.array([(row, h) for row in range(w.total_q) for h in range(w.num_q_heads)], np.int64)
    o_ref, lse_ref = lib().attention(pb, r.scale, items)
    compare(st.o.float().cpu().numpy().reshape(-1, w.head_dim), st.lse.cpu().numpy().T.reshape(-1), o_ref, lse_ref,
            "rope-decode-batch")
    ref = lib().token_mass(pb, r.scale)
    got = st.mass.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - ref) <= MASS_RTOL * np.abs(ref) + MASS_ATOL)


def test_fragment_prefill_is_bit_identical_under_page_permutation():
    w = SMALL["varlen-p16-g4"]()
    fr = _fragments(w, np.random.default_rng(63), per_seq=4)
    a = _run(w, frags=fr)
    b = _run(w, frags=fr, page_seed_offset=5)
    assert torch.equal(a.state[0].o, b.state[0].o) and torch.equal(a.state[0].lse, b.state[0].lse)
    assert torch.equal(a.state[0].mass, b.state[0].mass)


@pytest.mark.parametrize("name", ["varlen-p16-g4", "mha-d64-p128", "g16-p64"])
def test_realign_pass_then_plain_prefill_equals_gather_time_rope_bitwise(name):
    """segpaged_rope_realign into a second K pool + the plain prefill on it == the gather-time RoPE prefill."""
    from head_sparse_paged_b200 import segpaged as sp
    w = SMALL[name]()
    fr = _fragments(w, np.random.default_rng(64), per_seq=5)
    g = _run(w, frags=fr)
    r = Runner(w, keep_dense=True, split_ctas=g.split_ctas)
    st = r.state[0]
    k_out = torch.zeros_like(r.k_pool)
    fo, fs, fc = (torch.from_numpy(np.ascontiguousarray(x)).cuda() for x in fr)
    sp.segpaged_rope_realign(r.dims, r.cu_k_dev, r.ql_dev, st.cls_dev, st.table_dev, st.offs_dev, fo, fs, fc,
                             r.k_pool, k_out, r.status)
    sp.segpaged_attn_prefill(r.dims, st.q, k_out, r.v_pool, st.table_dev, st.units_dev, st.info, r.scale, st.o, st.lse,
                             r.workspace, r.status)
    torch.cuda.synchronize()
    r.check_status()
    assert torch.equal(st.o, g.state[0].o) and torch.equal(st.lse, g.state[0].lse)
    # the re-aligned pool itself: stored pages against the oracle's re-aligned keys
    k, v = r.dense[0]
    kn = orc.rope_fragment_keys(k.float().cpu().numpy(), w.cu_k(), *fr)
    c = w.classes[0]
    kp, _ = orc.build_pool(kn, v.float().cpu().numpy(), w.cu_k(), w.cu_q(), c[..., 0], c[..., 1], c[..., 2],
                           w.page_size, st.table, st.offs, r.num_pages)
    used = ~np.isnan(kp[:, 0, 0])
    np.testing.assert_array_equal(k_out.float().cpu().numpy()[used], kp[used])


def test_caller_level_rope_path_equals_gather_time_bitwise():
    """Runner.prefill_rope_auto takes the re-alignment pass on a layer whose query range spans several units per
    KV head, and returns the gather-time kernel's O and LSE bit for bit."""
    w = SMALL["g2-p64"]()
    fr = _fragments(w, np.random.default_rng(65), per_seq=6)
    g = _run(w, frags=fr)
    r = Runner(w, keep_dense=True, frags=fr, split_ctas=g.split_ctas)
    k_out = torch.zeros_like(r.k_pool)
    assert r.rope_realign_preferred()
    assert r.prefill_rope_auto(0, k_out) == "realign"
    torch.cuda.synchronize()
    r.check_status()
    assert torch.equal(r.state[0].o, g.state[0].o) and torch.equal(r.state[0].lse, g.state[0].lse)
