"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs.

Tolerance (the contract for fp32-accumulated outputs and final state):
relative Frobenius error <= 2e-3 and max-abs error <= 1e-2 x RMS(reference),
applied to o and to S_T.  The kernel feeds every derived operand to the
tensor core as a bf16 hi/lo pair (about 16 significant bits), so its error is
expected far below that; DESIGN_REL additionally guards that margin so a lost
lo term cannot hide behind the contract.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_linear_20_b200 import inputs

pytestmark = pytest.mark.gpu

REL_FRO = 2e-3
MAXABS_FRAC = 1e-2
DESIGN_REL = 1e-4

DEV = "cuda:0"


def _gdn():
    from gated_deltanet_linear_20_b200 import gdn
    return gdn


def errors(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300)
    rms = np.sqrt(np.mean(ref * ref)) if ref.size else 0.0
    mx = np.abs(got - ref).max() / max(rms, 1e-300) if ref.size else 0.0
    return float(rel), float(mx)


def assert_parity(got, ref, what, design=True):
    rel, mx = errors(got, ref)
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    assert rel <= REL_FRO and mx <= MAXABS_FRAC, f"{what}: rel_fro={rel:.3e} maxabs/rms={mx:.3e}"
    if design:
        assert rel <= DESIGN_REL, f"{what}: rel_fro={rel:.3e} above the hi/lo design margin"


def to_dev(d):
    return {k: (v.to(DEV) if v is not None else None) for k, v in d.items()}


def checked_prefill(q, k, v, g, beta, S0, chunk, **kw):
    """gdn.prefill with a device status word, which must stay 0 (no bounded
    device wait gave up)."""
    gdn = _gdn()
    status = torch.zeros(1, dtype=torch.int32, device=q.device)
    out = gdn.prefill(q, k, v, g, beta, S0, chunk=chunk, status=status, **kw)
    assert gdn.query_status(status) == 0, "a device-side wait timed out"
    return out


def gpu_prefill(d, chunk, S0=True, segmented=True):
    dd = to_dev(d)
    o, S_T = checked_prefill(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"],
                             dd["S0"] if S0 else None, chunk, segmented=segmented)
    return o.cpu().numpy(), S_T.cpu().numpy()


# gdn_prefill (one pass per chain) and gdn_prefill_ws (segments in parallel when
# the chains are too few to fill the GPU)
ENTRY = pytest.mark.parametrize("segmented", [False, True], ids=["single", "segmented"])


@pytest.mark.parametrize("chunk", [64, 16])
def test_tiny_b1_h2_t64(chunk):
    w = inputs.WORKLOADS["tiny_b1_h2_t64"]
    d = inputs.workload_inputs(w, seed=0)
    o, S_T = gpu_prefill(d, chunk)
    ro, rS = oracle.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    assert_parity(o, ro, "o")
    assert_parity(S_T, rS, "S_T")


@ENTRY
@pytest.mark.parametrize("chunk", [64, 16])
@pytest.mark.parametrize("T", [1, 15, 16, 17, 63, 64, 65, 100, 130, 200])
def test_ragged_lengths(T, chunk, segmented):
    d = inputs.prefill_inputs(2, T, 3, seed=T, s0_std=0.05)
    o, S_T = gpu_prefill(d, chunk, segmented=segmented)
    ro, rS = oracle.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    assert_parity(o, ro, f"o T={T}")
    assert_parity(S_T, rS, f"S_T T={T}")


@ENTRY
@pytest.mark.parametrize("chunk", [64, 16])
def test_prefill_b1_h16_t512(chunk, segmented):
    w = inputs.WORKLOADS["prefill_b1_h16_t512"]
    d = inputs.workload_inputs(w, seed=0)
    o, S_T = gpu_prefill(d, chunk, segmented=segmented)
    ro, rS = oracle.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    assert_parity(o, ro, "o")
    assert_parity(S_T, rS, "S_T")


@ENTRY
@pytest.mark.parametrize("chunk", [64, 16])
def test_prefill_b1_h16_t4096_carried_state(chunk, segmented):
    w = inputs.WORKLOADS["prefill_b1_h16_t4096_s0"]
    d = inputs.workload_inputs(w, seed=0)
    o, S_T = gpu_prefill(d, chunk, segmented=segmented)
    ro, rS = oracle.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    assert_parity(o, ro, "o")
    assert_parity(S_T, rS, "S_T")


@pytest.mark.parametrize("chunk", [64, 16])
def test_prefill_b4_h32_t32768_sampled_chains(chunk):
    """Full-size workload in the benchmark's launch configuration; the oracle
    recomputes a sample of (b, h) chains one by one."""
    w = inputs.WORKLOADS["prefill_b4_h32_t32768"]
    d = inputs.workload_inputs(w, seed=0, device=DEV)
    o, S_T = checked_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], chunk)
    for (b, h) in [(0, 0), (1, 17), (3, 31)]:
        sl = lambda x: x[b:b + 1, :, h:h + 1].cpu()
        ro, rS = oracle.prefill(sl(d["q"]), sl(d["k"]), sl(d["v"]), sl(d["g"]), sl(d["beta"]), None)
        assert_parity(o[b, :, h].cpu().numpy(), ro[0, :, 0], f"o chain ({b},{h})")
        assert_parity(S_T[b, h].cpu().numpy(), rS[0, 0], f"S_T chain ({b},{h})")
    del d, o, S_T
    torch.cuda.empty_cache()


@ENTRY
@pytest.mark.parametrize("chunk", [64, 16])
@pytest.mark.parametrize("g_mean", [0.0, 2.0])
def test_long_sequence_few_chains(chunk, g_mean, segmented):
    """2048 tokens on two chains: the chain and side warps drift furthest apart
    when few CTAs share the GPU, which is where hand-off bugs between tiles show."""
    d = inputs.prefill_inputs(1, 2048, 2, seed=21, g_mean=g_mean)
    o, S_T = gpu_prefill(d, chunk, S0=False, segmented=segmented)
    ro, rS = oracle.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], None)
    assert_parity(o, ro, f"o g_mean={g_mean}")
    assert_parity(S_T, rS, f"S_T g_mean={g_mean}")


@pytest.mark.parametrize("B,T,H,s0", [
    (1, 1000, 1, 0.05),    # one chain, 16 tiles: 8 segments of 2 tiles (7 chained ends)
    (1, 577, 3, 0.0),      # ragged last segment (one token in its last tile)
    (2, 700, 4, 0.1),      # 8 chains
    (1, 256, 37, 0.02),    # 37 chains: 2 segments of 2 tiles
])
@pytest.mark.parametrize("chunk", [64, 16])
def test_segmented_schedule_shapes(B, T, H, s0, chunk):
    gdn = _gdn()
    n, L, ws = gdn.schedule(B, T, H, torch.cuda.get_device_properties(0).multi_processor_count)
    assert n > 1, "shape meant to be segmented"
    assert gdn.workspace_bytes(B, T, H, chunk) == ws
    d = inputs.prefill_inputs(B, T, H, seed=T + H, s0_std=s0)
    o, S_T = gpu_prefill(d, chunk, S0=s0 > 0)
    ro, rS = oracle.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"] if s0 > 0 else None)
    assert_parity(o, ro, f"o {n}x{L}")
    assert_parity(S_T, rS, f"S_T {n}x{L}")


def test_segmented_in_place_state_deterministic_and_caller_workspace():
    gdn = _gdn()
    d = to_dev(inputs.prefill_inputs(1, 640, 4, seed=9, s0_std=0.05))
    assert gdn.workspace_bytes(1, 640, 4) > 0
    o_ref, S_ref = gdn.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    # S_T == S0 in place, with a caller-owned workspace reused twice
    ws = torch.empty(gdn.workspace_bytes(1, 640, 4), dtype=torch.uint8, device=DEV)
    for _ in range(2):
        S = d["S0"].clone()
        o, _ = gdn.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], S, S_T=S, workspace=ws)
        torch.cuda.synchronize()
        assert torch.equal(S, S_ref) and torch.equal(o, o_ref)


def test_segmented_workspace_errors():
    gdn = _gdn()
    d = to_dev(inputs.prefill_inputs(1, 640, 4, seed=9))
    need = gdn.workspace_bytes(1, 640, 4)
    with pytest.raises(gdn.GDNError) as e:
        gdn.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"],
                    workspace=torch.empty(need - 256, dtype=torch.uint8, device=DEV))
    assert e.value.code == gdn.GDN_ERR_WORKSPACE
    big = torch.empty(need + 512, dtype=torch.uint8, device=DEV)
    with pytest.raises(gdn.GDNError) as e:
        gdn.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], workspace=big[16:])
    assert e.value.code == gdn.GDN_ERR_WORKSPACE
    o = big[:1 * 640 * 4 * 128 * 4].view(torch.float32).view(1, 640, 4, 128)
    with pytest.raises(gdn.GDNError) as e:
        gdn.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], o=o, workspace=big)
    assert e.value.code == gdn.GDN_ERR_ALIAS


def packed(lengths, H, seed, s0_std=None, g_mean=0.0):
    """Packed inputs of sequences of the given lengths: per-sequence draws of
    the seeded generator, concatenated along tokens."""
    seqs = [inputs.prefill_inputs(1, L, H, seed=seed + i, g_mean=g_mean, s0_std=s0_std)
            for i, L in enumerate(lengths)]
    cat = lambda key: torch.cat([d[key][0] for d in seqs], 0)
    S0 = torch.cat([d["S0"] for d in seqs], 0) if s0_std else None
    cu = torch.tensor([0] + list(np.cumsum(lengths)), dtype=torch.int32)
    return seqs, dict(q=cat("q"), k=cat("k"), v=cat("v"), g=cat("g"), beta=cat("beta"), S0=S0, cu=cu)


@pytest.mark.parametrize("chunk", [64, 16])
@pytest.mark.parametrize("s0", [None, 0.05])
def test_varlen_packed_sequences(chunk, s0):
    """Packed sequences of mixed lengths (empty, 1 token, ragged, tile-aligned),
    each against the oracle run on that sequence alone."""
    lengths = [130, 0, 1, 64, 200, 17, 63, 65]
    H = 3
    seqs, pk = packed(lengths, H, seed=90, s0_std=s0)
    gdn = _gdn()
    dd = to_dev(pk)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, S_T = gdn.prefill_varlen(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["cu"], dd["S0"],
                                chunk=chunk, status=status)
    assert gdn.query_status(status) == 0
    o, S_T = o.cpu().numpy(), S_T.cpu().numpy()
    cu = pk["cu"].numpy()
    for n, d in enumerate(seqs):
        ro, rS = oracle.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
        if lengths[n]:
            assert_parity(o[cu[n]:cu[n + 1]], ro[0], f"o seq {n} (len {lengths[n]})")
        assert_parity(S_T[n], rS[0], f"S_T seq {n} (len {lengths[n]})") if (s0 or lengths[n]) else \
            np.testing.assert_array_equal(S_T[n], 0.0)


def test_varlen_equal_lengths_match_the_dense_call():
    """Equal lengths packed = the dense [B][T][H] call, bitwise (the same CTAs
    on the same tiles; only the token coordinates differ)."""
    B, T, H = 3, 150, 4
    d = to_dev(inputs.prefill_inputs(B, T, H, seed=8, s0_std=0.05))
    gdn = _gdn()
    o1, S1 = gdn.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], segmented=False)
    cu = torch.arange(0, (B + 1) * T, T, dtype=torch.int32, device=DEV)
    flat = lambda x: x.reshape(B * T, *x.shape[2:]).contiguous()
    o2, S2 = gdn.prefill_varlen(flat(d["q"]), flat(d["k"]), flat(d["v"]), flat(d["g"]),
                                flat(d["beta"]), cu, d["S0"])
    torch.cuda.synchronize()
    assert torch.equal(o1.reshape(B * T, H, 128), o2) and torch.equal(S1, S2)


@pytest.mark.parametrize("snap_every", [64, 128])
def test_varlen_state_snapshots(snap_every):
    """Snapshots after every snap_every tokens of each sequence equal the final
    state of the oracle run on that prefix."""
    lengths = [200, 64, 0, 129, 256]
    H = 2
    seqs, pk = packed(lengths, H, seed=55, s0_std=0.05)
    gdn = _gdn()
    dd = to_dev(pk)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, S_T, snaps = gdn.prefill_varlen(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["cu"],
                                       dd["S0"], status=status, snap_every=snap_every)
    assert gdn.query_status(status) == 0
    assert snaps.shape[0] == sum(L // snap_every for L in lengths)
    snaps = snaps.cpu().numpy()
    slot = 0
    for n, d in enumerate(seqs):
        for j in range(1, lengths[n] // snap_every + 1):
            t = j * snap_every
            cut = lambda x: x[:, :t]
            _, rS = oracle.prefill(cut(d["q"]), cut(d["k"]), cut(d["v"]), cut(d["g"]), cut(d["beta"]),
                                   d["S0"])
            assert_parity(snaps[slot], rS[0], f"snapshot {j} of seq {n} (t={t})")
            slot += 1
    # the dense outputs are unchanged by the snapshots
    o2, S2 = gdn.prefill_varlen(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["cu"], dd["S0"])
    torch.cuda.synchronize()
    assert torch.equal(o.cpu(), o2.cpu()) and torch.equal(S_T.cpu(), S2.cpu())


def test_varlen_bad_offsets_are_reported_on_the_device():
    _, pk = packed([40, 40], 2, seed=3)
    gdn = _gdn()
    dd = to_dev(pk)
    bad = torch.tensor([0, 50, 30], dtype=torch.int32, device=DEV)  # out of order
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    gdn.prefill_varlen(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], bad, status=status)
    assert gdn.query_status(status) == gdn.GDN_ERR_SHAPE


def test_varlen_malformed_offsets_leave_memory_before_the_snapshots_untouched():
    """cu_seqlens [100, 0, 200] with snapshots: sequence 0 ends before it
    starts.  Its own CTAs report GDN_ERR_SHAPE; sequence 1's snapshot slot base,
    which counts sequence 0's snapshots, would come out negative, so sequence 1
    takes no snapshots and nothing before the snapshot buffer is written."""
    H, T = 2, 200
    d = inputs.prefill_inputs(1, T, H, seed=91)
    gdn = _gdn()
    flat = lambda x: x[0].contiguous().to(DEV)
    cu = torch.tensor([100, 0, 200], dtype=torch.int32, device=DEV)
    guard = 2  # state-sized slots in front of the snapshot buffer
    buf = torch.full((guard + 3, H, 128, 128), 7.0, dtype=torch.float32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    gdn.prefill_varlen(flat(d["q"]), flat(d["k"]), flat(d["v"]), flat(d["g"]), flat(d["beta"]), cu,
                       status=status, snap_every=64, snaps=buf[guard:])
    assert gdn.query_status(status) == gdn.GDN_ERR_SHAPE
    assert torch.all(buf[:guard] == 7.0), "memory before the snapshot buffer was written"


def raw_qk(d, seed):
    """Un-normalised q, k (each token-head row scaled by a random factor in
    [0.2, 5]) and their fp64 L2-normalised versions."""
    rng = np.random.default_rng(seed)
    out = {}
    for key in ("q", "k"):
        x = d[key].double()
        scale = torch.from_numpy(rng.uniform(0.2, 5.0, size=x.shape[:-1] + (1,)))
        raw = (x * scale).to(torch.bfloat16)
        r64 = raw.double()
        out[key] = raw
        out[key + "_n"] = (r64 / torch.sqrt((r64 * r64).sum(-1, keepdim=True) + 1e-6))
    return out


@pytest.mark.parametrize("segmented", [False, True], ids=["single", "segmented"])
@pytest.mark.parametrize("chunk", [64, 16])
def test_fused_qk_l2norm_and_q_scale(chunk, segmented):
    """q / k L2 normalisation and the q scale fused into the kernel equal the
    oracle run on inputs normalised in fp64 beforehand."""
    d = inputs.prefill_inputs(1, 300, 6, seed=61, s0_std=0.05)
    r = raw_qk(d, 62)
    qs = 128 ** -0.5
    gdn = _gdn()
    dd = to_dev(d)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, S_T = gdn.prefill(r["q"].to(DEV), r["k"].to(DEV), dd["v"], dd["g"], dd["beta"], dd["S0"],
                         chunk=chunk, segmented=segmented, qk_l2norm=True, q_scale=qs, status=status)
    assert gdn.query_status(status) == 0
    ro, rS = oracle.prefill((r["q_n"] * qs).float(), r["k_n"].float(), d["v"], d["g"], d["beta"],
                            d["S0"])
    assert_parity(o.cpu().numpy(), ro, "o (fused norm)")
    assert_parity(S_T.cpu().numpy(), rS, "S_T (fused norm)")


@pytest.mark.parametrize("T", [1, 4])
def test_fused_qk_l2norm_in_decode(T):
    d = inputs.prefill_inputs(4, T, 8, seed=70 + T, s0_std=0.05)
    r = raw_qk(d, 71)
    qs = 0.5
    gdn = _gdn()
    dd = to_dev(d)
    S = dd["S0"].clone()
    o = gdn.decode_tokens(r["q"].to(DEV), r["k"].to(DEV), dd["v"], dd["g"], dd["beta"], S,
                          qk_l2norm=True, q_scale=qs)
    torch.cuda.synchronize()
    ro, rS = oracle.prefill((r["q_n"] * qs).float(), r["k_n"].float(), d["v"], d["g"], d["beta"],
                            d["S0"])
    assert_parity(o.cpu().numpy(), ro, f"o T={T}")
    assert_parity(S.cpu().numpy(), rS, f"S T={T}")


def test_default_options_are_bitwise_the_plain_call():
    import ctypes as ct
    gdn = _gdn()
    d = to_dev(inputs.prefill_inputs(2, 200, 3, seed=12, s0_std=0.02))
    o1, S1 = gdn.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], segmented=False)
    o2 = torch.empty_like(o1)
    S2 = torch.empty_like(S1)
    opts = gdn.Options(ct.sizeof(gdn.Options), 0, 1.0)
    rc = gdn.raw_prefill_ex(*[ct.c_void_p(t.data_ptr()) for t in (d["q"], d["k"], d["v"], d["g"],
                                                                    d["beta"], d["S0"], o2, S2)],
                            2, 200, 3, 128, 128, 64, None, ct.c_size_t(0), ct.byref(opts), None,
                            ct.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    assert rc == 0 and torch.equal(o1, o2) and torch.equal(S1, S2)


@pytest.mark.parametrize("pre", [False, True], ids=["plain", "qknorm"])
@pytest.mark.parametrize("chunk", [64, 16])
def test_bf16_o_is_the_fp32_o_rounded(chunk, pre):
    """o_bf16 stores the same fp32 o rounded to nearest even: bit for bit the
    fp32 call's o cast to bf16, with an identical end state.  T = 300 leaves a
    ragged last tile; a segmented request runs the single pass."""
    gdn = _gdn()
    d = to_dev(inputs.prefill_inputs(2, 300, 5, seed=81, s0_std=0.05))
    kw = dict(qk_l2norm=True, q_scale=0.25) if pre else {}
    o32, S32 = gdn.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], chunk=chunk,
                           segmented=False, **kw)
    for seg in (False, True):
        status = torch.zeros(1, dtype=torch.int32, device=DEV)
        o16, S16 = gdn.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], chunk=chunk,
                               segmented=seg, o_bf16=True, status=status, **kw)
        assert gdn.query_status(status) == 0
        assert o16.dtype == torch.bfloat16
        assert torch.equal(o16, o32.to(torch.bfloat16)), f"segmented={seg}"
        assert torch.equal(S16, S32), f"segmented={seg}"


@pytest.mark.parametrize("T", [1, 4])
def test_bf16_o_in_decode(T):
    gdn = _gdn()
    d = to_dev(inputs.prefill_inputs(8, T, 16, seed=90 + T, s0_std=0.05))
    S32 = d["S0"].clone()
    S16 = d["S0"].clone()
    if T == 1:
        sq = {n: d[n][:, 0] for n in ("q", "k", "v", "g", "beta")}
        o32 = gdn.decode_step(sq["q"], sq["k"], sq["v"], sq["g"], sq["beta"], S32)
        o16 = gdn.decode_step(sq["q"], sq["k"], sq["v"], sq["g"], sq["beta"], S16, o_bf16=True)
    else:
        o32 = gdn.decode_tokens(d["q"], d["k"], d["v"], d["g"], d["beta"], S32)
        o16 = gdn.decode_tokens(d["q"], d["k"], d["v"], d["g"], d["beta"], S16, o_bf16=True)
    torch.cuda.synchronize()
    assert o16.dtype == torch.bfloat16
    assert torch.equal(o16, o32.to(torch.bfloat16))
    assert torch.equal(S16, S32)


def test_bf16_o_full_size_against_the_oracle():
    """B1 H16 T512 with bf16 o: the oracle's fp64 o rounded to bf16 agrees to
    the rounding step (one bf16 ulp) plus the fp32 path's tolerance."""
    gdn = _gdn()
    d = inputs.workload_inputs(inputs.WORKLOADS["prefill_b1_h16_t512"], seed=0)
    dd = to_dev(d)
    o16, S = gdn.prefill(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["S0"], o_bf16=True)
    ro, rS = oracle.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    assert_parity(S.cpu().numpy(), rS, "S_T (bf16 o call)")
    got = o16.float().cpu().numpy().astype(np.float64)
    ref = np.asarray(ro, dtype=np.float64)
    ulp = np.abs(ref) * 2.0 ** -7            # one bf16 ulp at |ref| (8 significant bits)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    assert np.all(np.abs(got - ref) <= ulp + 1e-2 * rms)


def test_decode_b64_h16_256_steps_sampled_sequences():
    """256 in-place decode steps of the full batch on the GPU; sequences 0, 21,
    42, 63 (all 16 heads) checked against the oracle at every step."""
    w = inputs.WORKLOADS["decode_b64_h16"]
    d = inputs.workload_inputs(w, seed=0)
    dd = to_dev(d)
    S = dd["S"].clone()
    bsel = [0, 21, 42, 63]
    S_ref = d["S"][bsel].double().numpy()
    gdn = _gdn()
    worst = 0.0
    for t in range(w.decode_steps):
        o = gdn.decode_step(dd["q"][t], dd["k"][t], dd["v"][t], dd["g"][t], dd["beta"][t], S)
        ro, S_ref = oracle.decode_step(d["q"][t][bsel], d["k"][t][bsel], d["v"][t][bsel],
                                       d["g"][t][bsel], d["beta"][t][bsel], S_ref)
        got = o[bsel].cpu().numpy()
        assert_parity(got, ro, f"o step {t}")
        worst = max(worst, errors(got, ro)[0])
    assert_parity(S[bsel].cpu().numpy(), S_ref, "S after 256 steps")


@pytest.mark.parametrize("T", [1, 2, 3, 8, 16, 33])
def test_decode_tokens_against_oracle(T):
    """T tokens per sequence in one call, state in place: o at every token and
    the state after the burst against the oracle run from the same state."""
    d = inputs.prefill_inputs(4, T, 8, seed=40 + T, s0_std=0.05)
    dd = to_dev(d)
    gdn = _gdn()
    S = dd["S0"].clone()
    o = gdn.decode_tokens(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], S)
    torch.cuda.synchronize()
    ro, rS = oracle.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    assert_parity(o.cpu().numpy(), ro, f"o T={T}")
    assert_parity(S.cpu().numpy(), rS, f"S T={T}")


def test_decode_tokens_equals_repeated_steps():
    """A burst of 5 equals 5 single steps (the same per-token arithmetic, summed
    in another order by the burst kernel), and a burst of 1 is the step."""
    d = to_dev(inputs.prefill_inputs(3, 5, 4, seed=77, s0_std=0.05))
    gdn = _gdn()
    S1 = d["S0"].clone()
    o1 = gdn.decode_tokens(d["q"], d["k"], d["v"], d["g"], d["beta"], S1)
    S2 = d["S0"].clone()
    o2 = [gdn.decode_step(d["q"][:, t].contiguous(), d["k"][:, t].contiguous(),
                          d["v"][:, t].contiguous(), d["g"][:, t].contiguous(),
                          d["beta"][:, t].contiguous(), S2) for t in range(5)]
    torch.cuda.synchronize()
    assert_parity(S1.cpu().numpy(), S2.cpu().numpy(), "burst vs steps, S")
    assert_parity(o1.cpu().numpy(), torch.stack(o2, 1).cpu().numpy(), "burst vs steps, o")
    S3 = d["S0"].clone()
    o3 = gdn.decode_tokens(d["q"][:, :1].contiguous(), d["k"][:, :1].contiguous(),
                           d["v"][:, :1].contiguous(), d["g"][:, :1].contiguous(),
                           d["beta"][:, :1].contiguous(), S3)
    S4 = d["S0"].clone()
    o4 = gdn.decode_step(d["q"][:, 0].contiguous(), d["k"][:, 0].contiguous(),
                         d["v"][:, 0].contiguous(), d["g"][:, 0].contiguous(),
                         d["beta"][:, 0].contiguous(), S4)
    torch.cuda.synchronize()
    assert torch.equal(S3, S4) and torch.equal(o3[:, 0], o4)


def test_decode_equals_prefill_t1():
    d = inputs.prefill_inputs(3, 1, 5, seed=7, s0_std=0.1)
    dd = to_dev(d)
    gdn = _gdn()
    o_p, S_p = gdn.prefill(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["S0"], chunk=64)
    S = dd["S0"].clone()
    o_d = gdn.decode_step(dd["q"][:, 0], dd["k"][:, 0], dd["v"][:, 0], dd["g"][:, 0], dd["beta"][:, 0], S)
    torch.cuda.synchronize()
    assert_parity(o_d.cpu().numpy(), o_p[:, 0].cpu().numpy(), "decode vs prefill o")
    assert_parity(S.cpu().numpy(), S_p.cpu().numpy(), "decode vs prefill S")


@ENTRY
@pytest.mark.parametrize("chunk", [64, 16])
def test_split_carry(chunk, segmented):
    d = to_dev(inputs.prefill_inputs(1, 300, 4, seed=11, s0_std=0.05))
    gdn = _gdn()
    o, S_T = checked_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], chunk,
                             segmented=segmented)
    t1 = 130
    cut = lambda x, a, b: x[:, a:b].contiguous()
    o1, S1 = gdn.prefill(cut(d["q"], 0, t1), cut(d["k"], 0, t1), cut(d["v"], 0, t1),
                         cut(d["g"], 0, t1), cut(d["beta"], 0, t1), d["S0"], chunk=chunk,
                         segmented=segmented)
    o2, S2 = gdn.prefill(cut(d["q"], t1, 300), cut(d["k"], t1, 300), cut(d["v"], t1, 300),
                         cut(d["g"], t1, 300), cut(d["beta"], t1, 300), S1, chunk=chunk,
                         segmented=segmented)
    torch.cuda.synchronize()
    assert_parity(torch.cat([o1, o2], 1).cpu().numpy(), o.cpu().numpy(), "split o")
    assert_parity(S2.cpu().numpy(), S_T.cpu().numpy(), "split S_T")


def test_chunk16_agrees_with_chunk64():
    d = inputs.prefill_inputs(2, 257, 3, seed=5, s0_std=0.05)
    o64, S64 = gpu_prefill(d, 64)
    o16, S16 = gpu_prefill(d, 16)
    assert_parity(o16, o64, "o chunk16 vs 64")
    assert_parity(S16, S64, "S chunk16 vs 64")


@ENTRY
@pytest.mark.parametrize("chunk", [64, 16])
def test_bitwise_deterministic(chunk, segmented):
    d = to_dev(inputs.prefill_inputs(2, 333, 4, seed=3, s0_std=0.02))
    gdn = _gdn()
    a = gdn.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], chunk=chunk, segmented=segmented)
    b = gdn.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], chunk=chunk, segmented=segmented)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_zero_length_and_empty_batch():
    gdn = _gdn()
    d = to_dev(inputs.prefill_inputs(2, 0, 3, seed=1, s0_std=0.1))
    o, S_T = gdn.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], chunk=64)
    torch.cuda.synchronize()
    assert o.numel() == 0 and torch.equal(S_T, d["S0"])
    o, S_T = gdn.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], None, chunk=16)
    torch.cuda.synchronize()
    assert torch.count_nonzero(S_T) == 0
    e = to_dev(inputs.prefill_inputs(0, 10, 3, seed=1))
    o, S_T = gdn.prefill(e["q"], e["k"], e["v"], e["g"], e["beta"], None, chunk=64)
    assert o.numel() == 0 and S_T.numel() == 0


def test_in_place_state_and_status_word():
    gdn = _gdn()
    d = to_dev(inputs.prefill_inputs(1, 150, 2, seed=2, s0_std=0.1))
    o_ref, S_ref = gdn.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], chunk=64)
    S = d["S0"].clone()
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, S_out = gdn.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], S, chunk=64, S_T=S, status=status)
    assert gdn.query_status(status) == 0
    assert S_out.data_ptr() == S.data_ptr()
    assert torch.equal(S, S_ref) and torch.equal(o, o_ref)


def test_invariants_on_gpu():
    """beta = 0, g = 0 keeps S0; beta = 1 with exactly unit keys writes v (q = k)."""
    gdn = _gdn()
    d = inputs.prefill_inputs(1, 96, 2, seed=4, s0_std=0.1)
    d["beta"].zero_()
    d["g"].zero_()
    o, S_T = gpu_prefill(d, 64)
    assert_parity(S_T, d["S0"].double().numpy(), "S unchanged", design=False)
    ro = np.einsum("bhij,bthj->bthi", d["S0"].double().numpy(), d["q"].double().numpy())
    assert_parity(o, ro, "o = S0 q")
    rng = np.random.default_rng(4)
    k = np.zeros((1, 96, 2, 128), np.float32)
    for idx in np.ndindex(1, 96, 2):
        pos = rng.choice(128, 4, replace=False)
        k[idx][pos] = rng.choice([-0.5, 0.5], 4)
    e = inputs.prefill_inputs(1, 96, 2, seed=5)
    e["k"] = torch.from_numpy(k).to(torch.bfloat16)
    e["q"] = e["k"].clone()
    e["beta"].fill_(1.0)
    o, _ = gpu_prefill(e, 64, S0=False)
    assert_parity(o, e["v"].double().numpy(), "beta=1 writes v", design=False)


def test_rejects_unsupported_head_dim_on_gpu():
    gdn = _gdn()
    q = torch.zeros(1, 8, 1, 96, dtype=torch.bfloat16, device=DEV)
    g = torch.zeros(1, 8, 1, device=DEV)
    with pytest.raises(gdn.GDNError) as e:
        gdn.prefill(q, q, q, g, g)
    assert e.value.code == gdn.GDN_ERR_UNSUPPORTED
