"""The runner's CUDA-graph submission of the prefill call (Runner(graphs=True)), through the C ABI.

A graph replays the launches of one segpaged_attn_prefill call -- the work-counter clear when the plan has more
units than SMs, the persistent prefill kernel, and the combine kernel for split plans -- with the arguments of
the call it was captured from. Its O and LSE must be the direct call's bit for bit, step after step, while the step re-plans, re-uploads the plan and re-builds the pool into the same buffers; and on
the smallest case every row must also match the fp64 oracle.
"""
import numpy as np
import pytest
import torch

from head_sparse_paged_b200 import synth
from head_sparse_paged_b200.runner import Runner
from oracle import reference as orc

from gpu_common import compare, full_problem, oracle_dense

pytestmark = pytest.mark.gpu

# tiny: one kernel node; mistral-7b: split plan (prefill + combine), one unit per SM, no counter clear;
# llama-3.3-70b-decode32x16: more units than SMs (counter clear + prefill + combine)
CASES = ["tiny", "mistral-7b", "llama-3.3-70b-decode32x16"]


@pytest.mark.parametrize("name", CASES)
def test_graph_replay_equals_direct_call(name):
    w = synth.get(name)
    direct = Runner(w, graphs=False)
    direct.step()
    torch.cuda.synchronize()
    direct.check_status()
    o_ref, lse_ref = direct.state[0].o.clone(), direct.state[0].lse.clone()
    info = direct.state[0].info
    del direct
    torch.cuda.empty_cache()

    r = Runner(w, keep_dense=True, graphs=True)     # keep_dense: full_step rebuilds the pool from the dense K/V
    assert r.state[0].info == info
    side = torch.cuda.Stream()
    for it in range(3):
        st = r.state[0]
        st.o.fill_(float("nan"))
        st.lse.fill_(float("nan"))
        if it == 2:
            # replay on a caller stream, after the stream has seen the poisoning
            side.wait_stream(torch.cuda.current_stream())
            r.full_step(stream=side)
            torch.cuda.current_stream().wait_stream(side)
        else:
            r.full_step()
        torch.cuda.synchronize()
        r.check_status()
        assert r._prep_prefill[0][2] is not None, "the prefill call was not captured"
        assert torch.equal(st.o, o_ref) and torch.equal(st.lse, lse_ref), (name, it)


def test_graph_replay_matches_oracle_every_row():
    w = synth.get("tiny")
    r = Runner(w, keep_dense=True, graphs=True)
    r.step()
    r.step()          # the second call replays the graph captured by the first
    torch.cuda.synchronize()
    r.check_status()
    st = r.state[0]
    k, v = r.dense[0]
    qn, kn, vn = oracle_dense(w, st.q, k, v)
    items = np.array([(row, h) for row in range(w.total_q) for h in range(w.num_q_heads)], np.int64)
    o_ref, lse_ref = orc.OracleLib().attention(full_problem(w, 0, qn, kn, vn), r.scale, items)
    compare(st.o.float().cpu().numpy().reshape(-1, w.head_dim), st.lse.cpu().numpy().T.reshape(-1), o_ref, lse_ref,
            "graph tiny")
