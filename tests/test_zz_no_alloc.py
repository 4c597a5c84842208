"""The allocation-free prefill entry point (segpaged_attn_prefill_noalloc), through the C ABI.

It serves callers that cannot allocate device memory when they run prefill (code inside a framework's
own memory pool, or a runtime that forbids allocation on its request path): the unit list and the work
counter live in a static device array of the library instead of caller-provided memory. Two calls in a
row on each of two workloads must give what the workspace entry point gives, within the parity
tolerances; the second call reuses the array the first one left behind. This file is collected last.
"""
import numpy as np
import pytest
import torch

from head_sparse_paged_b200 import segpaged as sp
from head_sparse_paged_b200 import synth
from head_sparse_paged_b200.runner import Runner

pytestmark = pytest.mark.gpu

O_TOL, LSE_TOL = 1e-2, 1e-3


@pytest.mark.parametrize("name", ["mistral-7b", "tiny"])
def test_noalloc_prefill_matches_workspace_entry_point(name):
    w = synth.get(name)
    r = Runner(w, split_ctas=0)       # the allocation-free entry point takes plans without split units
    r.step()
    torch.cuda.synchronize()
    st = r.state[0]
    o_ref, lse_ref = st.o.clone(), st.lse.clone()
    for call in range(2):
        o = torch.full_like(st.o, float("nan"))
        lse = torch.full_like(st.lse, float("nan"))
        status = torch.zeros(1, dtype=torch.int32, device=o.device)
        sp.segpaged_attn_prefill_noalloc(r.dims, st.q, r.k_pool, r.v_pool, st.table_dev, st.units, r.scale, o, lse,
                                         status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
        eo = (o.float() - o_ref.float()).abs().max().item()
        el = (lse - lse_ref).abs().max().item()
        assert eo <= O_TOL and el <= LSE_TOL, (name, call, eo, el)


def test_noalloc_rejects_too_many_units():
    w = synth.tiny()
    dims = sp.Dims(1, 4, 2, 64, 16, 25)
    units = np.zeros((sp.NOALLOC_MAX_UNITS + 1, sp.UNIT_FIELDS), np.int32)
    dummy = torch.zeros(64, 4, 64, dtype=torch.bfloat16, device="cuda")
    pool = torch.zeros(25, 16, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(sp.SegPagedError) as e:
        sp.segpaged_attn_prefill_noalloc(dims, dummy, pool, pool, torch.zeros(25, dtype=torch.int32, device="cuda"),
                                         units, 0.125, torch.empty_like(dummy),
                                         torch.empty(4, 64, dtype=torch.float32, device="cuda"))
    assert e.value.code == -6
