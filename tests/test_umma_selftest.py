"""GPU check of the tcgen05 building blocks the prefill kernel relies on: each
MMA form (K-major / MN-major SW128 descriptors for A and for B, A from tensor
memory, N=16 sub-block with row and K offsets, negated A, N=64) on one 128x128 tile
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
@pytest.mark.parametrize("mode", [0, 1, 2, 3, 4, 5, 6, 7, 8])
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
    elif mode == 5:
        ref, got = Af @ Bf[:64].T, D.double().cpu()[:, :64]
    elif mode == 6:
        ref, got = Af.T @ Bf[:64].T, D.double().cpu()[:, :64]
    elif mode == 7:
        ref, got = Af[:64].T @ Bf[:64, :64].T, D.double().cpu()[:, :64]
    else:
        ref, got = Af @ Bf[:, :64], D.double().cpu()[:, :64]
    err = (got - ref).abs().max().item()
    assert err < 1e-3 * max(1.0, ref.abs().max().item()), f"mode {mode}: max err {err}"


@pytest.mark.gpu
def test_mma_issue_rate():
    """Issue cost of tcgen05.mma (printed with -s): the kernel design counts MMA
    instructions, not only FLOPs, so this records how long a run of 128 MMAs of
    M = 128 and N = 32..256 takes to issue and to complete, on one CTA and on
    one CTA per SM; with one accumulator, with four rotating accumulators, and
    split between two issuing warps.  Checks only that every run completes."""
    lib = ctypes.CDLL(build_selftest())
    lib.umma_issue_probe.argtypes = [ctypes.c_int] * 3 + [ctypes.c_void_p] * 3
    lib.umma_issue_probe.restype = ctypes.c_int
    dev = torch.device("cuda:0")
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    out = torch.zeros(2 * sms, dtype=torch.int64, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    n = 128
    modes = list(range(8)) + [8, 9, 11, 16, 17, 19]  # + rotating accumulators, two issuers
    for mode in modes:
        N = [64, 128, 256, 32][mode & 3]
        for ctas in (1, sms):
            for _ in range(2):  # the second run is the one recorded
                rc = lib.umma_issue_probe(mode, n, ctas, out.data_ptr(), status.data_ptr(),
                                          torch.cuda.current_stream().cuda_stream)
                assert rc == 0
            torch.cuda.synchronize()
            assert int(status.item()) == 0
            t = out.view(sms, 2)[:ctas].double().cpu().mean(0)
            tflops = 128 * N * 16 * 2 * n / (t[1].item() * 1e-9) / 1e12
            kind = "two issuers" if mode & 16 else "4 accumulators" if mode & 8 else "one accumulator"
            print(f"A from {'TMEM' if mode & 4 else 'SMEM'}, {kind}, N={N:3d} CTAs={ctas:3d}: "
                  f"issue {t[0].item() / n:.1f} ns/MMA, complete {t[1].item() / n:.1f} ns/MMA, "
                  f"{tflops:.2f} TFLOP/s per SM")
