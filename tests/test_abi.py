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
    for n in ("gdn_prefill", "gdn_prefill_ws", "gdn_prefill_varlen", "gdn_prefill_workspace_bytes",
              "gdn_prefill_schedule", "gdn_prefill_ex", "gdn_decode_step", "gdn_decode_tokens",
              "gdn_decode_ex", "gdn_kda_prefill", "gdn_kda_decode", "gdn_abi_version",
              "gdn_status_str", "gdn_query_status"):
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
    assert gdn.abi_version() == 8
    for code in range(-9, 1):
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
    (dict(Dk=96), -4), (dict(Dv=512), -4), (dict(chunk=32), -4), (dict(chunk=0), -4),
    (dict(q=None), -1), (dict(o=None), -1), (dict(S_T=None), -1), (dict(g=None), -1),
    (dict(q=P + 8), -2), (dict(o=P + 0x40000004), -2), (dict(g=P + 0x30000002), -2),
    (dict(S0=P + 0x60000008), -2),
    (dict(o=P + 0x10000000 + 0x100), -5),                # o overlaps k
    (dict(S0=P + 0x50000000 + 0x40), -5),                 # S0 partially overlaps S_T
    (dict(S_T=P + 0x20000000 + 0x1000), -5),              # S_T overlaps v
    (dict(S_T=P + 0x31000000 - 0x100), -5),               # S_T runs into beta
    (dict(B=1 << 16, T=1 << 16, H=1), -3),                # too many elements
], ids=lambda x: str(x))
def test_prefill_rejects_bad_arguments(gdn, over, code):
    assert gdn.raw_prefill(*prefill_args(**over)) == code


def test_prefill_empty_batch_is_a_noop(gdn):
    assert gdn.raw_prefill(*prefill_args(B=0, q=None, k=None, o=None, S_T=None)) == 0
    assert gdn.raw_prefill(*prefill_args(H=0)) == 0


@pytest.mark.parametrize("over,code", [
    (dict(B=-1), -3), (dict(Dk=96), -4), (dict(chunk=32), -4), (dict(q=None), -1),
    (dict(q=P + 8), -2), (dict(o=P + 0x10000000 + 0x100), -5),
], ids=lambda x: str(x))
def test_prefill_ws_rejects_bad_arguments_like_prefill(gdn, over, code):
    a = prefill_args(**over)
    assert gdn.raw_prefill_ws(*(a[:14] + [None, 0] + a[14:])) == code


def test_prefill_ws_empty_batch_is_a_noop(gdn):
    a = prefill_args(B=0, q=None, k=None, o=None, S_T=None)
    assert gdn.raw_prefill_ws(*(a[:14] + [None, 0] + a[14:])) == 0


def test_workspace_query_is_zero_without_a_device_or_for_bad_sizes(gdn):
    import torch
    assert gdn.workspace_bytes(1, 512, 16, chunk=32) == 0
    assert gdn.workspace_bytes(-1, 512, 16) == 0
    if not torch.cuda.is_available():
        assert gdn.workspace_bytes(1, 512, 16) == 0


def plan_cost(tiles, n, L):
    # the time model documented with the planner (units: one single-pass tile)
    return tiles if n == 1 else 1.2 * L + 0.4 * (n - 1) + 0.6


@pytest.mark.parametrize("B,T,H,expect", [
    (1, 64, 2, (1, 1)),           # one tile: nothing to cut
    (1, 512, 16, (4, 2)),         # 16 chains x 8 tiles: 4 segments of 2 tiles
    (1, 4096, 16, (5, 13)),       # 16 chains x 64 tiles: 2*5-1 = 9 CTAs per chain
    (4, 32768, 32, (1, 512)),     # 128 chains already fill the GPU
    (1, 100, 16, (1, 2)),         # 2 tiles: segmenting does not pay
])
def test_schedule_of_the_benchmark_shapes(gdn, B, T, H, expect):
    n, L, ws = gdn.schedule(B, T, H, 148)
    assert (n, L) == expect
    tiles = (T + 63) // 64
    if n == 1:
        assert ws == 0 and L == tiles
    else:
        assert (n - 1) * L < tiles <= n * L               # every segment is non-empty
        assert B * H * (2 * n - 1) <= 148                 # first launch fits in one wave
        f_bytes = B * T * H * 128 * 4
        assert ws == ((f_bytes + 255) // 256) * 256 + 2 * B * H * n * 128 * 128 * 4
        # the planner took the cheapest admissible segment count
        nmax = (148 // (B * H) + 1) // 2
        costs = []
        for m in range(1, min(nmax, tiles) + 1):
            Lm = -(-tiles // m)
            mm = -(-tiles // Lm)
            costs.append(plan_cost(tiles, mm, Lm))
        assert abs(plan_cost(tiles, n, L) - min(costs)) < 1e-9


def test_schedule_rejects_bad_sizes(gdn):
    with pytest.raises(gdn.GDNError):
        gdn.schedule(-1, 64, 1, 148)
    assert gdn.schedule(1, 512, 16, 0)[0] == 1     # no multiprocessor count: single pass
    assert gdn.schedule(0, 512, 16, 148)[0] == 1


def varlen_args(**over):
    a = dict(q=P, k=P + 0x10000000, v=P + 0x20000000, g=P + 0x30000000, beta=P + 0x31000000,
             S0=None, o=P + 0x40000000, S_T=P + 0x50000000, cu=P + 0x60000000, N=3, total_T=200,
             H=2, Dk=128, Dv=128, chunk=64, snaps=None, snap_every=0, n_snaps=0, status=None,
             stream=None)
    a.update(over)
    return [a[k] for k in ("q", "k", "v", "g", "beta", "S0", "o", "S_T", "cu", "N", "total_T",
                           "H", "Dk", "Dv", "chunk", "snaps", "snap_every", "n_snaps", "status",
                           "stream")]


@pytest.mark.parametrize("over,code", [
    (dict(N=-1), -3), (dict(total_T=-1), -3), (dict(Dk=256), -4), (dict(Dv=32), -4),
    (dict(chunk=8), -4),
    (dict(cu=None), -1), (dict(S_T=None), -1), (dict(q=None), -1),
    (dict(cu=P + 0x60000002), -2), (dict(o=P + 0x40000008), -2),
    (dict(o=P + 0x60000000 - 64), -5),          # o runs into cu_seqlens
    (dict(S_T=P + 0x60000000 - 64 * 1024), -5),  # S_T runs into cu_seqlens
    (dict(S_T=P + 0x10000000), -5),              # S_T over k
    (dict(snaps=P + 0x70000000, snap_every=100, n_snaps=2), -4),   # not a multiple of 64
    (dict(snaps=P + 0x70000000, snap_every=0, n_snaps=2), -4),
    (dict(snaps=P + 0x70000008, snap_every=64, n_snaps=2), -2),
    (dict(snaps=P + 0x50000000, snap_every=64, n_snaps=2), -5),    # snapshots over S_T
    (dict(n_snaps=-1), -3),
], ids=lambda x: str(x))
def test_prefill_varlen_rejects_bad_arguments(gdn, over, code):
    assert gdn.raw_prefill_varlen(*varlen_args(**over)) == code


@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64), (128, 256), (64, 256)])
def test_prefill_varlen_other_head_dims_pass_validation(gdn, dk, dv):
    """Packed sequences run on the chunked tensor-core kernel at every Dk of 64
    or 128: valid calls pass validation (then fail only for want of a device)."""
    assert gdn.raw_prefill_varlen(*varlen_args(Dk=dk, Dv=dv)) not in VALIDATION_CODES + (0,)


def test_prefill_varlen_overlap_checks_follow_the_head_dims(gdn):
    """3 sequences x 2 heads of 128 x 256 fp32 states take 768 KiB: an S_T that
    starts 768 KiB - 16 B before cu_seqlens runs into it, at 128 x 128 it does not."""
    s_t = P + 0x60000000 - 6 * 128 * 256 * 4 + 16
    assert gdn.raw_prefill_varlen(*varlen_args(S_T=s_t, Dk=128, Dv=256)) == -5
    assert gdn.raw_prefill_varlen(*varlen_args(S_T=s_t)) not in VALIDATION_CODES + (0,)


def test_prefill_varlen_no_sequences_is_a_noop(gdn):
    assert gdn.raw_prefill_varlen(*varlen_args(N=0, q=None, S_T=None)) == 0


def test_options_struct_matches_the_header(gdn):
    import ctypes as ct
    text = open(HEADER).read()
    assert "typedef struct gdn_options" in text
    assert ct.sizeof(gdn.Options) == 16
    assert [f[0] for f in gdn.Options._fields_] == ["size", "qk_l2norm", "q_scale", "o_bf16"]


def test_invalid_options_are_rejected(gdn):
    import ctypes as ct
    short = gdn.Options(4, 1, 1.0)                     # size smaller than the struct
    nan = gdn.Options(ct.sizeof(gdn.Options), 0, float("nan"))
    for opts in (short, nan):
        a = prefill_args()
        assert gdn.raw_prefill_ex(*(a[:14] + [None, 0, ct.byref(opts)] + a[14:])) == -4
        d = decode_tokens_args()
        assert gdn.raw_decode_ex(*(d[:12] + [ct.byref(opts)] + d[12:])) == -4


def test_bf16_o_overlap_uses_two_byte_elements(gdn):
    """With o_bf16 o spans B*T*H*Dv*2 bytes: an o that would run into S_T as
    fp32 (64 KiB) stops short of it as bf16 (32 KiB)."""
    import ctypes as ct
    o = P + 0x50000000 - 48 * 1024
    a = prefill_args(o=o)
    plain = gdn.Options(ct.sizeof(gdn.Options), 0, 1.0, 0)
    half = gdn.Options(ct.sizeof(gdn.Options), 0, 1.0, 1)
    assert gdn.raw_prefill_ex(*(a[:14] + [None, 0, ct.byref(plain)] + a[14:])) == -5
    assert gdn.raw_prefill_ex(*(a[:14] + [None, 0, ct.byref(half)] + a[14:])) not in (0, -5)


def test_options_without_o_bf16_field_are_accepted(gdn):
    """A 12-byte struct (before o_bf16) reads as o_bf16 = 0: the fp32 overlap
    rule applies, so the call fails on the overlap and not on the size."""
    import ctypes as ct
    a = prefill_args(o=P + 0x50000000 - 48 * 1024)
    old = gdn.Options(12, 0, 1.0, 1)   # the trailing o_bf16 lies past `size`: ignored
    assert gdn.raw_prefill_ex(*(a[:14] + [None, 0, ct.byref(old)] + a[14:])) == -5


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


def decode_tokens_args(**over):
    a = dict(q=P, k=P + 0x1000000, v=P + 0x2000000, g=P + 0x3000000, beta=P + 0x3100000,
             S=P + 0x4000000, o=P + 0x8000000, B=2, T=4, H=3, Dk=128, Dv=128, status=None,
             stream=None)
    a.update(over)
    return [a[k] for k in ("q", "k", "v", "g", "beta", "S", "o", "B", "T", "H", "Dk", "Dv",
                           "status", "stream")]


@pytest.mark.parametrize("over,code", [
    (dict(T=-1), -3), (dict(B=-1), -3), (dict(Dv=32), -4), (dict(k=None), -1),
    (dict(o=P + 0x8000004), -2), (dict(o=P + 0x4000000 + 64), -5),
    (dict(v=P + 0x4000000 + 4096), -5),     # v overlaps the state
], ids=lambda x: str(x))
def test_decode_tokens_rejects_bad_arguments(gdn, over, code):
    assert gdn.raw_decode_tokens(*decode_tokens_args(**over)) == code


def test_decode_tokens_empty_is_a_noop(gdn):
    assert gdn.raw_decode_tokens(*decode_tokens_args(T=0)) == 0
    assert gdn.raw_decode_tokens(*decode_tokens_args(B=0)) == 0


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


# ---------------------------------------------------------------------------- KDA entry points

def kda_args(**over):
    # B=1 T=64 H=2: q/k/v 32 KiB each, g 64 KiB, o 64 KiB, state 128 KiB
    a = dict(q=P, k=P + 0x1000000, v=P + 0x2000000, g=P + 0x3000000, beta=P + 0x3100000,
             S0=P + 0x4000000, o=P + 0x5000000, S_T=P + 0x6000000, B=1, T=64, H=2, Dk=128,
             Dv=128, status=None, stream=None)
    a.update(over)
    return [a[k] for k in ("q", "k", "v", "g", "beta", "S0", "o", "S_T", "B", "T", "H", "Dk",
                           "Dv", "status", "stream")]


@pytest.mark.parametrize("over,code", [
    (dict(B=-1), -3), (dict(T=-1), -3), (dict(Dk=96), -4), (dict(Dv=512), -4),
    (dict(S_T=None), -1), (dict(q=None), -1), (dict(g=None), -1), (dict(o=None), -1),
    (dict(g=P + 0x3000004), -2),                  # g rows are copied in 16-byte pieces
    (dict(S_T=P + 0x6000008), -2), (dict(o=P + 0x5000002), -2),
    (dict(S0=P + 0x6000000 + 0x1000), -5),        # S0 partly overlaps S_T
    (dict(o=P + 0x3000000 + 0x100), -5),           # o over g
    (dict(S_T=P + 0x2000000 + 0x40), -5),          # S_T over v
    (dict(o=P + 0x6000000 - 0x100), -5),           # o runs into S_T
], ids=lambda x: str(x))
def test_kda_prefill_rejects_bad_arguments(gdn, over, code):
    assert gdn.raw_kda_prefill(*kda_args(**over)) == code


def test_kda_no_op_shapes_return_ok_without_a_device(gdn):
    assert gdn.raw_kda_prefill(*kda_args(B=0)) == 0
    assert gdn.raw_kda_prefill(*kda_args(H=0, q=None, S_T=None)) == 0
    # T = 0 in place has nothing to do; T = 0 to another buffer copies (needs the device)
    assert gdn.raw_kda_prefill(*kda_args(T=0, S0=P + 0x6000000)) == 0
    assert gdn.raw_kda_prefill(*kda_args(T=0)) not in (0, -1, -2, -3, -4, -5)


def test_kda_in_place_state_is_accepted_by_validation(gdn):
    """S0 == S_T is the decode form: validation passes it (the call then fails
    only for want of a device)."""
    rc = gdn.raw_kda_prefill(*kda_args(S0=P + 0x6000000))
    assert rc not in (-1, -2, -3, -4, -5)


def test_kda_decode_argument_checks(gdn):
    d = dict(q=P, k=P + 0x1000000, v=P + 0x2000000, g=P + 0x3000000, beta=P + 0x3100000,
             S=P + 0x4000000, o=P + 0x5000000, B=4, T=1, H=2, Dk=128, Dv=128, status=None,
             stream=None)
    order = ("q", "k", "v", "g", "beta", "S", "o", "B", "T", "H", "Dk", "Dv", "status", "stream")
    call = lambda **o: gdn.raw_kda_decode(*[{**d, **o}[k] for k in order])
    assert call(S=None) == -1
    assert call(B=-2) == -3
    assert call(Dk=100) == -4
    assert call(o=P + 0x4000000 + 0x10) == -5      # o inside the state
    assert call(B=0) == 0


# ---------------------------------------------------------------------------- other head dims

VALIDATION_CODES = (-1, -2, -3, -4, -5)


@pytest.mark.parametrize("dk,dv", [(64, 64), (256, 256), (128, 256), (64, 128), (256, 64)])
def test_other_head_dims_pass_validation(gdn, dk, dv):
    """Head dims 64, 128, 256 in any combination are accepted by gdn_prefill,
    the decode entry points and the KDA ones (without a device the calls then
    fail at the device check, not at validation)."""
    assert gdn.raw_prefill(*prefill_args(Dk=dk, Dv=dv)) not in VALIDATION_CODES + (0,)
    d = decode_args(Dk=dk, Dv=dv)
    assert gdn.raw_decode_step(*d) not in VALIDATION_CODES + (0,)
    assert gdn.raw_kda_prefill(*kda_args(Dk=dk, Dv=dv)) not in VALIDATION_CODES + (0,)
    assert gdn.workspace_bytes(1, 4096, 16, 64, dk, dv) == 0 or (dk, dv) == (128, 128)
    a = prefill_args(Dk=dk, Dv=dv)
    assert gdn.raw_prefill_ws(*(a[:14] + [None, 0] + a[14:])) not in VALIDATION_CODES + (0,)
    assert gdn.raw_prefill_static_ws(*a) not in VALIDATION_CODES + (0, -9)  # no scratch needed
    t = decode_tokens_args(Dk=dk, Dv=dv)
    assert gdn.raw_decode_tokens(*t) not in VALIDATION_CODES + (0,)
    kd = [P, P + 0x1000000, P + 0x2000000, P + 0x3000000, P + 0x3100000, P + 0x4000000,
          P + 0x5000000, 4, 2, 2, dk, dv, None, None]
    assert gdn.raw_kda_decode(*kd) not in VALIDATION_CODES + (0,)


@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64), (128, 256)])
def test_fused_options_pass_validation_on_the_tensor_core_dims(gdn, dk, dv):
    """Prefill with Dk = 64 or 128 runs the chunked tensor-core kernel, which has
    the fused q/k norm, q scale and bf16 o: valid options pass validation (and
    then fail only for want of a device)."""
    import ctypes as ct
    for opts in (gdn.Options(ct.sizeof(gdn.Options), 1, 0.5, 0), gdn.Options(ct.sizeof(gdn.Options), 0, 1.0, 1)):
        a = prefill_args(Dk=dk, Dv=dv)
        assert gdn.raw_prefill_ex(*(a[:14] + [None, 0, ct.byref(opts)] + a[14:])) not in VALIDATION_CODES + (0,)


def test_row_kernel_dims_reject_fused_options(gdn):
    """The row kernel (prefill with Dk = 256; decode outside 64 x 64 and
    128 x 128) has no fused options; the 64 x 64 decode has them."""
    import ctypes as ct
    opts = gdn.Options(ct.sizeof(gdn.Options), 1, 1.0, 0)
    a = prefill_args(Dk=256, Dv=256)
    assert gdn.raw_prefill_ex(*(a[:14] + [None, 0, ct.byref(opts)] + a[14:])) == -4
    for dk, dv in ((256, 256), (64, 128), (128, 64)):
        d = decode_tokens_args(Dk=dk, Dv=dv)
        assert gdn.raw_decode_ex(*(d[:12] + [ct.byref(opts)] + d[12:])) == -4
    d = decode_tokens_args(Dk=64, Dv=64)
    assert gdn.raw_decode_ex(*(d[:12] + [ct.byref(opts)] + d[12:])) not in VALIDATION_CODES + (0,)


def test_other_head_dims_size_the_overlap_checks(gdn):
    """Byte extents follow Dk and Dv: with Dv = 256, an o that starts 32 KiB
    before S_T (64 token-heads x 1 KiB) overlaps it; with Dv = 64 it does not."""
    o = P + 0x50000000 - 0x8000
    assert gdn.raw_prefill(*prefill_args(o=o, Dk=64, Dv=256)) == -5
    assert gdn.raw_prefill(*prefill_args(o=o, Dk=64, Dv=64)) not in VALIDATION_CODES


def test_plain_c_client_links_and_gets_the_documented_codes(gdn, tmp_path):
    """tests/csrc/abi_c_client.c includes include/gdn.h as C99 (gcc, -Werror),
    links the library and checks the device-free entry points and the
    validation codes of the compute entry points."""
    lib_dir = os.path.dirname(gdn.library_path)
    exe = str(tmp_path / "abi_c_client")
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                           os.path.join(ROOT, "tests", "csrc", "abi_c_client.c"), "-L", lib_dir, "-lgdn_b200",
                           "-Wl,-rpath," + lib_dir, "-o", exe])
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "0 failure(s)" in r.stdout


def test_kda_options_validation(gdn):
    """gdn_kda_prefill_ex / gdn_kda_decode_ex: the fused norm, q scale and bf16
    o exist with Dk = 128 in the prefill, and at 128 x 128 and 64 x 64 in
    decode; elsewhere, and for invalid structs, GDN_ERR_UNSUPPORTED; valid
    options where they exist pass validation (then fail only for want of a
    device)."""
    import ctypes as ct
    good = gdn.Options(ct.sizeof(gdn.Options), 1, 0.5, 0)
    bf16 = gdn.Options(ct.sizeof(gdn.Options), 0, 1.0, 1)
    short = gdn.Options(4, 1, 1.0, 0)
    a = kda_args()
    ins = lambda args, o: args[:13] + [ct.byref(o)] + args[13:]
    assert gdn.raw_kda_prefill_ex(*ins(a, good)) not in (0, -1, -2, -3, -4, -5)
    assert gdn.raw_kda_prefill_ex(*ins(a, bf16)) not in (0, -1, -2, -3, -4, -5)
    assert gdn.raw_kda_prefill_ex(*ins(kda_args(Dk=64, Dv=64), bf16)) == -4
    assert gdn.raw_kda_prefill_ex(*ins(a, short)) == -4
    assert gdn.raw_kda_prefill_ex(*ins(kda_args(Dk=64, Dv=64), good)) == -4
    for dv in (64, 256):  # Dk = 128: the tensor-core kernel, with the options
        assert gdn.raw_kda_prefill_ex(*ins(kda_args(Dv=dv), good)) not in (0, -1, -2, -3, -4, -5)
    assert gdn.raw_kda_prefill_ex(*(a[:13] + [None] + a[13:])) not in (0, -1, -2, -3, -4, -5)
    d = [P, P + 0x1000000, P + 0x2000000, P + 0x3000000, P + 0x3100000, P + 0x4000000,
         P + 0x5000000, 4, 1, 2, 128, 128]
    tail = [None, None]
    assert gdn.raw_kda_decode_ex(*(d + [ct.byref(good)] + tail)) not in (0, -1, -2, -3, -4, -5)
    assert gdn.raw_kda_decode_ex(*(d + [ct.byref(bf16)] + tail)) not in (0, -1, -2, -3, -4, -5)
    assert gdn.raw_kda_decode_ex(*(d[:10] + [64, 128] + [ct.byref(bf16)] + tail)) == -4
    d64 = d[:10] + [64, 64]
    assert gdn.raw_kda_decode_ex(*(d64 + [ct.byref(good)] + tail)) not in (0, -1, -2, -3, -4, -5)
    assert gdn.raw_kda_decode_ex(*(d64 + [None] + tail)) not in (0, -1, -2, -3, -4, -5)
    d64x128 = d[:10] + [64, 128]
    assert gdn.raw_kda_decode_ex(*(d64x128 + [ct.byref(good)] + tail)) == -4


def kda_varlen_args(**over):
    # N=3 sequences, total_T=200, H=2, Dk=128: q/k 100 KiB each, g 200 KiB, o 200 KiB (Dv 128)
    a = dict(q=P, k=P + 0x1000000, v=P + 0x2000000, g=P + 0x3000000, beta=P + 0x3100000,
             S0=None, o=P + 0x5000000, S_T=P + 0x6000000, cu=P + 0x7000000, N=3, total_T=200,
             H=2, Dk=128, Dv=128, snaps=None, snap_every=0, n_snaps=0, status=None, stream=None)
    a.update(over)
    return [a[k] for k in ("q", "k", "v", "g", "beta", "S0", "o", "S_T", "cu", "N", "total_T",
                           "H", "Dk", "Dv", "snaps", "snap_every", "n_snaps", "status", "stream")]


@pytest.mark.parametrize("over,code", [
    (dict(N=-1), -3), (dict(total_T=-1), -3), (dict(H=-1), -3),
    (dict(Dk=64, Dv=64), -4), (dict(Dk=256), -4), (dict(Dv=32), -4),
    (dict(cu=None), -1), (dict(S_T=None), -1), (dict(q=None), -1), (dict(g=None), -1),
    (dict(cu=P + 0x7000002), -2), (dict(g=P + 0x3000004), -2), (dict(o=P + 0x5000008), -2),
    (dict(S_T=P + 0x6000008), -2),
    (dict(S0=P + 0x6000000 + 0x1000), -5),         # S0 partly overlaps S_T
    (dict(o=P + 0x3000000 + 0x100), -5),           # o over g
    (dict(o=P + 0x7000000 - 64), -5),              # o runs into cu_seqlens
    (dict(S_T=P + 0x7000000 - 64 * 1024), -5),     # S_T runs into cu_seqlens
    (dict(S_T=P + 0x2000000 + 0x40), -5),          # S_T over v
    (dict(n_snaps=-1), -3),
    (dict(snaps=P + 0x8000000, snap_every=48, n_snaps=2), -4),    # not a multiple of 32
    (dict(snaps=P + 0x8000000, snap_every=0, n_snaps=2), -4),
    (dict(snaps=P + 0x8000008, snap_every=32, n_snaps=2), -2),
    (dict(snaps=P + 0x6000000, snap_every=32, n_snaps=2), -5),    # snapshots over S_T
    (dict(snaps=P + 0x7000000 - 1024, snap_every=32, n_snaps=1), -5),  # into cu_seqlens
], ids=lambda x: str(x))
def test_kda_prefill_varlen_rejects_bad_arguments(gdn, over, code):
    assert gdn.raw_kda_prefill_varlen(*kda_varlen_args(**over)) == code


@pytest.mark.parametrize("dv", [64, 128, 256])
def test_kda_prefill_varlen_valid_calls_pass_validation(gdn, dv):
    """Dk = 128 with Dv 64, 128 or 256 passes validation (the call then fails
    only for want of a device); no sequences or no heads is a no-op."""
    assert gdn.raw_kda_prefill_varlen(*kda_varlen_args(Dv=dv)) not in VALIDATION_CODES + (0,)
    assert gdn.raw_kda_prefill_varlen(*kda_varlen_args(
        Dv=dv, snaps=P + 0x8000000, snap_every=32, n_snaps=6)) not in VALIDATION_CODES + (0,)
    assert gdn.raw_kda_prefill_varlen(*kda_varlen_args(N=0, q=None, S_T=None)) == 0
    assert gdn.raw_kda_prefill_varlen(*kda_varlen_args(H=0, cu=None)) == 0


def test_packed_calls_take_the_pre_step_options(gdn):
    """gdn_prefill_varlen_ex and gdn_kda_prefill_varlen_ex accept qk_l2norm,
    q_scale and o_bf16 (the call then fails only for want of a device), reject a
    short struct and a NaN scale (GDN_ERR_UNSUPPORTED), and validate every other
    argument as the calls without options do (o sized by its element type)."""
    import ctypes as ct
    good = ct.byref(gdn.Options(ct.sizeof(gdn.Options), 1, 0.5, 1))
    bad = [ct.byref(gdn.Options(4, 1, 1.0)),
           ct.byref(gdn.Options(ct.sizeof(gdn.Options), 0, float("nan")))]
    with_opts = lambda a, o: a[:18] + [o] + a[18:]
    for dk, dv in ((128, 128), (64, 64), (128, 256)):
        a = varlen_args(Dk=dk, Dv=dv)
        assert gdn.raw_prefill_varlen_ex(*with_opts(a, good)) not in VALIDATION_CODES + (0,)
        assert gdn.raw_prefill_varlen_ex(*with_opts(a, None)) not in VALIDATION_CODES + (0,)
        for o in bad:
            assert gdn.raw_prefill_varlen_ex(*with_opts(a, o)) == -4
    assert gdn.raw_prefill_varlen_ex(*with_opts(varlen_args(N=-1), good)) == -3
    assert gdn.raw_prefill_varlen_ex(*with_opts(varlen_args(S_T=P + 0x10000000), good)) == -5
    kwith = lambda a, o: a[:17] + [o] + a[17:]
    for dv in (64, 128, 256):
        a = kda_varlen_args(Dv=dv)
        assert gdn.raw_kda_prefill_varlen_ex(*kwith(a, good)) not in VALIDATION_CODES + (0,)
        for o in bad:
            assert gdn.raw_kda_prefill_varlen_ex(*kwith(a, o)) == -4
    assert gdn.raw_kda_prefill_varlen_ex(*kwith(kda_varlen_args(Dk=64, Dv=64), good)) == -4
    assert gdn.raw_kda_prefill_varlen_ex(*kwith(kda_varlen_args(cu=None), good)) == -1
    # 200 tokens x 2 heads x 128: o runs 200 KiB as fp32, 100 KiB as bf16
    plain = ct.byref(gdn.Options(ct.sizeof(gdn.Options), 0, 1.0, 0))
    o = P + 0x7000000 - 128 * 1024                # 128 KiB before cu_seqlens
    assert gdn.raw_kda_prefill_varlen_ex(*kwith(kda_varlen_args(o=o), plain)) == -5
    assert gdn.raw_kda_prefill_varlen_ex(*kwith(kda_varlen_args(o=o), good)) not in VALIDATION_CODES + (0,)
