"""A pipeline wait that never completes gives up after its limit, reports SEGPAGED_STATUS_TIMEOUT in the
status word and returns, and the CUDA context keeps working. The wait is the same bounded mbarrier wait
the prefill kernel uses; nothing ever arrives on the barrier (no fault, trap or hang is provoked)."""
import ctypes
import os
import subprocess
import time

import pytest
import torch

from head_sparse_paged_b200 import segpaged as sp

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(HERE, "csrc", "libwait_timeout_probe.so")


def build_probe() -> str:
    src = os.path.join(HERE, "csrc", "wait_timeout_probe.cu")
    if not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(src):
        subprocess.check_call(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O2", "-std=c++17",
                               "-Xcompiler", "-fPIC", "-shared", "-o", LIB, src])
    return LIB


def test_bounded_wait_times_out_and_reports():
    lib = ctypes.CDLL(build_probe())
    lib.segpaged_test_wait_timeout.restype = ctypes.c_int
    lib.segpaged_test_wait_timeout.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_uint64]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    result = torch.zeros(3, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.time()
    rc = lib.segpaged_test_wait_timeout(ctypes.c_void_p(status.data_ptr()), ctypes.c_void_p(result.data_ptr()),
                                        20_000_000)   # 20 ms
    elapsed = time.time() - t0
    assert rc == 0
    assert int(status.item()) == sp.STATUS_TIMEOUT
    assert result.tolist() == [0, 1, 1]     # wait gave up, abort flag raised, later kernel ran
    assert elapsed < 5.0
    assert torch.ones(4, device="cuda").sum().item() == 4.0   # torch work still runs on the context
