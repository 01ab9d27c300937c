"""Failure detection without a GPU fault: the bounded mbarrier wait that every
kernel uses gives up after its limit on a phase that never completes, reports
GDN_ERR_DEVICE_TIMEOUT through the device status word, and the context stays
usable (a normal prefill runs right after)."""
from __future__ import annotations

import ctypes
import os
import subprocess

import pytest
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "csrc", "wait_selftest.cu")
LIB = os.path.join(HERE, "csrc", "libwait_selftest.so")
GDN_ERR_DEVICE_TIMEOUT = -7


def build_wait_selftest(force: bool = False) -> str:
    deps = [SRC, os.path.join(ROOT, "gated_deltanet_linear_20_b200", "csrc", "sm100.cuh")]
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < max(map(os.path.getmtime, deps)):
        from gated_deltanet_linear_20_b200.build import nvcc, ARCH_FLAGS
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.check_call([nvcc(), *ARCH_FLAGS, "-O2", "-std=c++17", "-Xcompiler", "-fPIC",
                               "-shared", "-cudart", "static",
                               "-I" + os.path.join(ROOT, "gated_deltanet_linear_20_b200", "csrc"),
                               SRC, "-o", tmp])
        os.replace(tmp, LIB)
    return LIB


def test_wait_selftest_library_builds():
    assert os.path.exists(build_wait_selftest())


def _run(mode, limit_ns):
    lib = ctypes.CDLL(build_wait_selftest())
    lib.wait_selftest.argtypes = [ctypes.c_int, ctypes.c_ulonglong] + [ctypes.c_void_p] * 4
    lib.wait_selftest.restype = ctypes.c_int
    dev = torch.device("cuda:0")
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    elapsed = torch.zeros(1, dtype=torch.int64, device=dev)
    left = torch.zeros(1, dtype=torch.int32, device=dev)
    rc = lib.wait_selftest(mode, limit_ns, status.data_ptr(), elapsed.data_ptr(), left.data_ptr(),
                           torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert rc == 0
    return int(status.item()), int(elapsed.item()), int(left.item())


@pytest.mark.gpu
def test_wait_that_never_completes_gives_up_and_reports():
    status, elapsed, left = _run(0, 1_000_000)           # 1 ms limit
    assert status == GDN_ERR_DEVICE_TIMEOUT
    assert 1_000_000 <= elapsed < 1_000_000_000
    assert left == 1


@pytest.mark.gpu
def test_completed_phase_returns_at_once():
    status, elapsed, left = _run(1, 1_000_000)
    assert status == 0 and elapsed < 1_000_000 and left == 1


@pytest.mark.gpu
def test_role_leaves_together_after_a_timeout_and_the_context_stays_usable():
    status, _, left = _run(2, 2_000_000)
    assert status == GDN_ERR_DEVICE_TIMEOUT
    assert left == 128                                    # every thread of the role left
    # the context still runs real work correctly
    from gated_deltanet_linear_20_b200 import gdn, inputs
    import oracle
    import numpy as np
    d = inputs.prefill_inputs(1, 70, 2, seed=5)
    dd = {k: (v.cuda() if v is not None else None) for k, v in d.items()}
    st = torch.zeros(1, dtype=torch.int32, device="cuda:0")
    o, S_T = gdn.prefill(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], status=st)
    assert gdn.query_status(st) == 0
    ro, _ = oracle.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"])
    assert np.linalg.norm(o.cpu().numpy() - ro) <= 2e-3 * np.linalg.norm(ro)
