"""segpaged_build on the GPU against the oracle's pool gather: bit-exact, with and without RoPE."""
import numpy as np
import pytest
import torch

from head_sparse_paged_b200 import segpaged as sp
from head_sparse_paged_b200 import synth
from head_sparse_paged_b200.runner import Runner
from oracle import reference as orc


pytestmark = pytest.mark.gpu

CASES = {
    "tiny": lambda: synth.tiny(),
    "mistral-7b-rope": lambda: synth.mistral_7b(),
    "edge-p16-rope": lambda: synth.custom("edge-p16-rope", [(1000, 300), (37, 37), (5, 0), (129, 1)], 8, 2, 128, 16,
                                          [[(0, 0, 100), (1, 0, 0)], [(0, 50, 3), (0, 2, 1)], [(1, 0, 0), (0, 1, 1)],
                                           [(0, 128, 1), (1, 0, 0)]], seed=7, rope_theta=1e4,
                                          rope_deltas=[17, 0, 4095, 1]),
    "edge-d64-p128": lambda: synth.custom("edge-d64-p128", [(300, 300), (130, 2)], 8, 8, 64, 128,
                                          [[(0, 5, 17), (0, 0, 1), (1, 0, 0), (0, 300, 300), (0, 1000, 2), (0, 64, 64),
                                            (0, 127, 129), (0, 3, 250)]] * 2, seed=8, page_order="interleaved"),
}


@pytest.mark.parametrize("name", list(CASES))
def test_build_bit_exact(name):
    w = CASES[name]()
    r = Runner(w, keep_dense=True)
    torch.cuda.synchronize()
    r.check_status()
    st = r.state[0]
    k, v = r.dense[0]
    c = st.cls
    # the oracle gathers from the un-rotated dense K and applies its own RoPE table and rule per page
    k_raw = k.float().cpu().numpy()
    vn = v.float().cpu().numpy()
    rope = orc.rope_cos_sin(w.rope_theta, w.rope_deltas, w.head_dim) if w.rope_theta is not None else None
    kp, vp = orc.build_pool(k_raw, vn, w.cu_k(), w.cu_q(), c[..., 0], c[..., 1], c[..., 2], w.page_size, st.table,
                            st.offs, r.num_pages, rope_cs=rope)
    used = np.unique(st.table)
    gk = r.k_pool.float().cpu().numpy()[used]
    gv = r.v_pool.float().cpu().numpy()[used]
    np.testing.assert_array_equal(gk.view(np.uint32), kp[used].view(np.uint32))
    np.testing.assert_array_equal(gv.view(np.uint32), vp[used].view(np.uint32))


def test_build_reports_bad_page_id():
    w = synth.tiny()
    dims = sp.Dims(1, 4, 2, 64, 16, 30)
    cls = w.classes[0]
    _, _, per = sp.segpaged_pages_bytes(dims, w.ctx_lens, w.q_lens, cls)
    table, offs, n = synth.assign_pages(per.reshape(1, 2), "shuffled", 3)
    table[5] = 30                                    # one past the pool: the kernel must skip and report it
    q, k, v = synth.layer_inputs(w, 0, device="cuda")
    kp = torch.zeros(30, 16, 64, dtype=torch.bfloat16, device="cuda")
    vp = torch.zeros_like(kp)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    sp.segpaged_build(dims, k, v, torch.from_numpy(w.cu_k()).cuda(), torch.tensor(w.q_lens, dtype=torch.int32).cuda(),
                      torch.from_numpy(cls.reshape(-1)).cuda(), torch.from_numpy(table).cuda(),
                      torch.from_numpy(offs).cuda(), None, kp, vp, status)
    torch.cuda.synchronize()
    assert int(status.item()) & sp.STATUS_PAGE_ID
