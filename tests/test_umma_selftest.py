"""GPU check of the tcgen05 building blocks the prefill kernel relies on: each
MMA form (K-major / MN-major SW128 descriptors, A from tensor memory, N=16
sub-block with row and K offsets, negated A, N=64) on one 128x128 tile
against a host matmul of the same bf16 inputs."""
from __future__ import annotations

import ctypes
import os
import subprocess

import pytest
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "csrc", "umma_selftest.cu")
LIB = os.path.join(HERE, "csrc", "libumma_selftest.so")


def build_selftest(force: bool = False) -> str:
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < max(
            os.path.getmtime(SRC),
            os.path.getmtime(os.path.join(ROOT, "gated_deltanet_linear_20_b200", "csrc", "sm100.cuh"))):
        from gated_deltanet_linear_20_b200.build import nvcc, ARCH_FLAGS
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.check_call([nvcc(), *ARCH_FLAGS, "-O2", "-std=c++17", "-Xcompiler", "-fPIC",
                               "-shared", "-cudart", "static",
                               "-I" + os.path.join(ROOT, "gated_deltanet_linear_20_b200", "csrc"),
                               SRC, "-o", tmp])
        os.replace(tmp, LIB)
    return LIB


def test_selftest_library_builds():
    assert os.path.exists(build_selftest())


@pytest.mark.gpu
@pytest.mark.parametrize("mode", [0, 1, 2, 3, 4, 5])
def test_umma_forms(mode):
    lib = ctypes.CDLL(build_selftest())
    lib.umma_selftest.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
    lib.umma_selftest.restype = ctypes.c_int
    gen = torch.Generator().manual_seed(100 + mode)
    A = torch.randn(128, 128, generator=gen).to(torch.bfloat16)
    B = torch.randn(128, 128, generator=gen).to(torch.bfloat16)
    dev = torch.device("cuda:0")
    Ad, Bd = A.to(dev), B.to(dev)
    D = torch.zeros(128, 128, dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    rc = lib.umma_selftest(Ad.data_ptr(), Bd.data_ptr(), D.data_ptr(), mode, status.data_ptr(),
                           torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert rc == 0 and int(status.item()) == 0
    Af, Bf = A.double(), B.double()
    if mode in (0, 2):
        ref, got = Af @ Bf.T, D.double().cpu()
    elif mode == 1:
        ref, got = Af @ Bf, D.double().cpu()
    elif mode == 3:
        ref, got = Af[:, 16:32] @ Bf[32:48, 16:32].T, D.double().cpu()[:, :16]
    elif mode == 4:
        ref, got = 1.0 - Af @ Bf.T, D.double().cpu()
    else:
        ref, got = Af @ Bf[:64].T, D.double().cpu()[:, :64]
    err = (got - ref).abs().max().item()
    assert err < 1e-3 * max(1.0, ref.abs().max().item()), f"mode {mode}: max err {err}"
