"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function include/gdn.h declares, and rejects bad arguments with the
documented codes before touching a device."""
from __future__ import annotations

import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdn.h")


@pytest.fixture(scope="module")
def gdn():
    from gated_deltanet_linear_20_b200 import build
    build.build()
    from gated_deltanet_linear_20_b200 import gdn as mod
    return mod


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(gdn_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("gdn_prefill", "gdn_decode_step", "gdn_abi_version", "gdn_status_str",
              "gdn_query_status"):
        assert n in names


def test_library_exports_every_declared_symbol(gdn):
    lib = ctypes.CDLL(gdn.library_path)
    for name in declared_functions():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", gdn.library_path], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (gdn_\w+)", out))
    assert set(declared_functions()) <= exported


def test_abi_version_and_status_strings(gdn):
    assert gdn.abi_version() == 1
    for code in range(-7, 1):
        s = gdn.status_str(code)
        assert s and s != "unknown status code"
    assert gdn.status_str(12345) == "unknown status code"


P = 0x100000  # a fake, 16-byte aligned "device" address: validation never dereferences it


def prefill_args(**over):
    a = dict(q=P, k=P + 0x10000000, v=P + 0x20000000, g=P + 0x30000000, beta=P + 0x31000000,
             S0=None, o=P + 0x40000000, S_T=P + 0x50000000, B=1, T=64, H=2, Dk=128, Dv=128,
             chunk=64, status=None, stream=None)
    a.update(over)
    return [a[k] for k in ("q", "k", "v", "g", "beta", "S0", "o", "S_T", "B", "T", "H", "Dk", "Dv",
                           "chunk", "status", "stream")]


@pytest.mark.parametrize("over,code", [
    (dict(B=-1), -3), (dict(T=-5), -3), (dict(H=-2), -3),
    (dict(Dk=64), -4), (dict(Dv=256), -4), (dict(chunk=32), -4), (dict(chunk=0), -4),
    (dict(q=None), -1), (dict(o=None), -1), (dict(S_T=None), -1), (dict(g=None), -1),
    (dict(q=P + 8), -2), (dict(o=P + 0x40000004), -2), (dict(g=P + 0x30000002), -2),
    (dict(S0=P + 0x60000008), -2),
    (dict(o=P + 0x10000000 + 0x100), -5),                # o overlaps k
    (dict(S0=P + 0x50000000 + 0x40), -5),                 # S0 partially overlaps S_T
    (dict(B=1 << 16, T=1 << 16, H=1), -3),                # too many elements
], ids=lambda x: str(x))
def test_prefill_rejects_bad_arguments(gdn, over, code):
    assert gdn.raw_prefill(*prefill_args(**over)) == code


def test_prefill_empty_batch_is_a_noop(gdn):
    assert gdn.raw_prefill(*prefill_args(B=0, q=None, k=None, o=None, S_T=None)) == 0
    assert gdn.raw_prefill(*prefill_args(H=0)) == 0


def decode_args(**over):
    a = dict(q=P, k=P + 0x1000000, v=P + 0x2000000, g=P + 0x3000000, beta=P + 0x3100000,
             S=P + 0x4000000, o=P + 0x8000000, B=2, H=3, Dk=128, Dv=128, status=None, stream=None)
    a.update(over)
    return [a[k] for k in ("q", "k", "v", "g", "beta", "S", "o", "B", "H", "Dk", "Dv", "status",
                           "stream")]


@pytest.mark.parametrize("over,code", [
    (dict(B=-1), -3), (dict(Dk=96), -4), (dict(S=None), -1), (dict(o=None), -1),
    (dict(S=P + 0x4000004), -2), (dict(o=P + 0x4000000 + 64), -5), (dict(q=P + 0x4000000 + 64), -5),
], ids=lambda x: str(x))
def test_decode_rejects_bad_arguments(gdn, over, code):
    assert gdn.raw_decode_step(*decode_args(**over)) == code


def test_decode_empty_batch_is_a_noop(gdn):
    assert gdn.raw_decode_step(*decode_args(B=0)) == 0


def test_valid_call_without_a_gpu_reports_no_launch(gdn):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    # valid arguments reach the device check, which fails cleanly on a CPU-only host
    assert gdn.raw_prefill(*prefill_args()) in (-6, -4)
    assert gdn.raw_decode_step(*decode_args()) in (-6, -4)


def test_tensor_binding_refuses_cpu_tensors(gdn):
    import torch
    q = torch.zeros(1, 4, 1, 128, dtype=torch.bfloat16)
    g = torch.zeros(1, 4, 1)
    with pytest.raises(ValueError):
        gdn.prefill(q, q, q, g, g)
    with pytest.raises(ValueError):
        gdn.decode_step(q[:, 0], q[:, 0], q[:, 0], g[:, 0], g[:, 0], torch.zeros(1, 1, 128, 128))
