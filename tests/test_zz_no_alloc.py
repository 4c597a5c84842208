"""The allocation-free prefill entry point (segpaged_attn_prefill_noalloc), through the C ABI.

It serves callers that cannot allocate device memory when they run prefill (code inside a framework's
own memory pool, or a runtime that forbids allocation on its request path): the unit list and the work
counter live in a static device array of the library instead of caller-provided memory.

It runs the same kernel variant on the same plan as segpaged_attn_prefill, so its O and LSE must be the
workspace entry point's bit for bit, and within the parity tolerances of the fp64 oracle on every row.
Calls run back to back, the later ones on a plan with fewer units than the array still holds from the
earlier ones, so a unit left behind by an earlier call would show. The first plan has more units than
the GPU has SMs, so its CTAs claim units from the array's work counter, which the call clears; the
others have one unit per CTA and leave the counter alone. This file is collected last.
"""
import numpy as np
import pytest
import torch

from head_sparse_paged_b200 import segpaged as sp
from head_sparse_paged_b200 import synth
from head_sparse_paged_b200.runner import Runner
from oracle import reference as orc

from gpu_common import compare, full_problem, oracle_dense

pytestmark = pytest.mark.gpu


# 160 half units (80 sequences x 2 KV heads, 20-64 query rows each): more units than SMs
MANY = [(200 + (53 * i) % 190, 20 + (7 * i) % 45) for i in range(80)]


def _workload(name):
    if name == "many-units":
        return synth.custom(name, MANY, 4, 2, 128, 16, [[(1, 0, 0), (0, 16, 64)]] * len(MANY), seed=31)
    return synth.get(name)


def _setup(name):
    w = _workload(name)
    r = Runner(w, split_ctas=0, keep_dense=True)   # the allocation-free entry point takes plans without split units
    r.step()
    torch.cuda.synchronize()
    r.check_status()
    st = r.state[0]
    k, v = r.dense[0]
    qn, kn, vn = oracle_dense(w, st.q, k, v)
    items = np.array([(row, h) for row in range(w.total_q) for h in range(w.num_q_heads)], np.int64)
    o_ref, lse_ref = orc.OracleLib().attention(full_problem(w, 0, qn, kn, vn), r.scale, items)
    return w, r, st.o.clone(), st.lse.clone(), o_ref, lse_ref


def test_noalloc_prefill_matches_workspace_entry_point_and_oracle():
    cases = {name: _setup(name) for name in ("many-units", "mistral-7b", "tiny")}
    units = {name: len(c[1].state[0].units) for name, c in cases.items()}
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert units["tiny"] < units["mistral-7b"] < sms < units["many-units"], units
    # calls on ever smaller plans, each over the array the larger plans before it filled
    for name in ("many-units", "many-units", "mistral-7b", "mistral-7b", "tiny", "tiny"):
        w, r, o_ws, lse_ws, o_ref, lse_ref = cases[name]
        st = r.state[0]
        o = torch.full_like(st.o, float("nan"))
        lse = torch.full_like(st.lse, float("nan"))
        status = torch.zeros(1, dtype=torch.int32, device=o.device)
        sp.segpaged_attn_prefill_noalloc(r.dims, st.q, r.k_pool, r.v_pool, st.table_dev, st.units, r.scale, o, lse,
                                         status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0, name
        assert torch.equal(o, o_ws) and torch.equal(lse, lse_ws), name
        compare(o.float().cpu().numpy().reshape(-1, w.head_dim), lse.cpu().numpy().T.reshape(-1), o_ref, lse_ref,
                f"noalloc {name}")


def test_noalloc_rejects_too_many_units():
    dims = sp.Dims(1, 4, 2, 64, 16, 25)
    units = np.zeros((sp.NOALLOC_MAX_UNITS + 1, sp.UNIT_FIELDS), np.int32)
    q = torch.zeros(64, 4, 64, dtype=torch.bfloat16, device="cuda")
    pool = torch.zeros(25, 16, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(sp.SegPagedError) as e:
        sp.segpaged_attn_prefill_noalloc(dims, q, pool, pool, torch.zeros(25, dtype=torch.int32, device="cuda"),
                                         units, 0.125, torch.empty_like(q),
                                         torch.empty(4, 64, dtype=torch.float32, device="cuda"))
    assert e.value.code == -6
