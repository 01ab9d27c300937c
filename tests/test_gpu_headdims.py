"""GPU parity at head dims other than 128 x 128 (64, 128, 256 in any
combination, Dk != Dv included), through the same C entry points, against the
fp64 oracles (which take any Dk, Dv).  Prefill with Dk = 64 or 128 runs the
chunked tensor-core kernel (Dv = 256: two CTAs per chain, 128 state rows each;
Dv = 64: one CTA with its upper 64 rows held at zero); decode at 64 x 64 runs
the streaming decode kernel (two 256-byte rows per warp-wide load); Dk = 256,
the other decode dims and the per-channel-gate prefill run the row-parallel
fp32 kernel.  The contract and the
1e-4 design margin are those of the other tests.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_linear_20_b200 import inputs
from tests.test_gpu_parity import DEV, assert_parity, raw_qk, to_dev

pytestmark = pytest.mark.gpu

DIMS = [(64, 64), (256, 256), (128, 256), (256, 128), (64, 128), (128, 64), (64, 256)]


def _gdn():
    from gated_deltanet_linear_20_b200 import gdn
    return gdn


@pytest.mark.parametrize("dk,dv", DIMS, ids=lambda x: str(x))
@pytest.mark.parametrize("BH", [(1, 3), (4, 16)], ids=["16rows", "32rows"])
def test_prefill_other_head_dims(dk, dv, BH):
    """Scalar gate through gdn.prefill (gdn_prefill_ws): T = 77 is not a
    multiple of any staging chunk; S0 is carried in."""
    B, H = BH
    T = 77 if B == 1 else 33
    d = inputs.prefill_inputs(B, T, H, dk, dv, seed=dk + dv + B, s0_std=0.05)
    dd = to_dev(d)
    o, S_T = _gdn().prefill(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["S0"])
    torch.cuda.synchronize()
    ro, rS = oracle.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    assert_parity(o.cpu().numpy(), ro, f"o {dk}x{dv}")
    assert_parity(S_T.cpu().numpy(), rS, f"S_T {dk}x{dv}")


@pytest.mark.parametrize("dk,dv", [(64, 64), (256, 256), (128, 256)], ids=lambda x: str(x))
def test_long_prefill_other_head_dims(dk, dv):
    d = inputs.prefill_inputs(1, 1024, 2, dk, dv, seed=3, g_mean=2.0, s0_std=0.02)
    dd = to_dev(d)
    o, S_T = _gdn().prefill(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["S0"], chunk=16,
                            segmented=False)
    torch.cuda.synchronize()
    ro, rS = oracle.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    assert_parity(o.cpu().numpy(), ro, f"o {dk}x{dv} T1024")
    assert_parity(S_T.cpu().numpy(), rS, f"S_T {dk}x{dv} T1024")


@pytest.mark.parametrize("dk,dv", [(64, 64), (256, 256), (128, 256), (256, 64)], ids=lambda x: str(x))
def test_decode_other_head_dims(dk, dv):
    """Five single-token steps (the direct path) and a 3-token burst (the
    staged path), the state in place, against the oracle over all 8 tokens."""
    d = inputs.prefill_inputs(16, 8, 4, dk, dv, seed=dk * 3 + dv, s0_std=0.05)
    dd = to_dev(d)
    gdn = _gdn()
    S = dd["S0"].clone()
    step = lambda sl: [dd[key][:, sl].contiguous() for key in ("q", "k", "v", "g", "beta")]
    outs = [gdn.decode_step(*step(t), S) for t in range(5)]
    o3 = gdn.decode_tokens(*step(slice(5, 8)), S)
    torch.cuda.synchronize()
    ro, rS = oracle.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    o = torch.cat([torch.stack(outs, 1), o3], 1).cpu().numpy()
    assert_parity(o, ro, f"o decode {dk}x{dv}")
    assert_parity(S.cpu().numpy(), rS, f"S decode {dk}x{dv}")


def test_decode_64_b64_h16_steps():
    """The 64 x 64 decode at 64 x 16 heads: 6 single-token steps and a 3-token
    burst on every head, the state in place, against the oracle; then the same
    inputs again give the same bits."""
    d = inputs.prefill_inputs(64, 9, 16, 64, 64, seed=64, s0_std=0.02)
    dd = to_dev(d)
    gdn = _gdn()
    step = lambda sl: [dd[key][:, sl].contiguous() for key in ("q", "k", "v", "g", "beta")]

    def run():
        S = dd["S0"].clone()
        outs = [gdn.decode_step(*step(t), S).unsqueeze(1) for t in range(6)]
        outs.append(gdn.decode_tokens(*step(slice(6, 9)), S))
        torch.cuda.synchronize()
        return torch.cat(outs, 1), S
    o, S = run()
    ro, rS = oracle.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    assert_parity(o.cpu().numpy(), ro, "o decode 64x64 B64 H16")
    assert_parity(S.cpu().numpy(), rS, "S decode 64x64 B64 H16")
    o2, S2 = run()
    assert torch.equal(o, o2) and torch.equal(S, S2), "not bitwise run-to-run"


@pytest.mark.parametrize("dk,dv", [(64, 64), (256, 256), (128, 64), (64, 256), (128, 256)], ids=lambda x: str(x))
def test_kda_other_head_dims(dk, dv):
    d = inputs.kda_inputs(2, 50, 3, dk, dv, seed=dk + 2 * dv, s0_std=0.05)
    dd = to_dev(d)
    gdn = _gdn()
    o, S_T = gdn.kda_prefill(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["S0"])
    S = dd["S0"].clone()
    o1 = gdn.kda_decode(*[dd[key][:, 0].contiguous() for key in ("q", "k", "v", "g", "beta")], S)
    torch.cuda.synchronize()
    ro, rS = oracle.kda_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    assert_parity(o.cpu().numpy(), ro, f"o kda {dk}x{dv}")
    assert_parity(S_T.cpu().numpy(), rS, f"S_T kda {dk}x{dv}")
    assert_parity(o1.cpu().numpy(), ro[:, 0], f"o kda decode {dk}x{dv}")


def test_other_head_dims_in_place_and_deterministic():
    gdn = _gdn()
    d = to_dev(inputs.prefill_inputs(2, 40, 3, 256, 64, seed=21, s0_std=0.05))
    o1, S1 = gdn.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    o2, S2 = gdn.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    S_in = d["S0"].clone()
    o3, S3 = gdn.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], S_in, S_T=S_in)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(S1, S2)
    assert torch.equal(o3, o1) and torch.equal(S3, S1) and S3.data_ptr() == S_in.data_ptr()


TC_DIMS = [(64, 64), (64, 128), (64, 256), (128, 64), (128, 256)]


@pytest.mark.parametrize("dk,dv", TC_DIMS, ids=lambda x: str(x))
@pytest.mark.parametrize("chunk", [64, 16])
@pytest.mark.parametrize("T", [1, 64, 130], ids=lambda t: f"T{t}")
def test_tensor_core_head_dims_chunks_and_tails(dk, dv, chunk, T):
    """The tensor-core shapes at both chunks, one token, one full tile and a
    ragged third tile; S0 carried in; the device status word stays 0."""
    gdn = _gdn()
    d = inputs.prefill_inputs(2, T, 3, dk, dv, seed=dk + dv + T + chunk, s0_std=0.05)
    dd = to_dev(d)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, S_T = gdn.prefill(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["S0"], chunk=chunk,
                         status=status)
    assert gdn.query_status(status) == 0
    ro, rS = oracle.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    assert_parity(o.cpu().numpy(), ro, f"o {dk}x{dv} chunk {chunk} T {T}")
    assert_parity(S_T.cpu().numpy(), rS, f"S_T {dk}x{dv} chunk {chunk} T {T}")


@pytest.mark.parametrize("dk,dv", [(128, 256), (64, 64)], ids=lambda x: str(x))
def test_tensor_core_head_dims_in_place_deterministic_and_segmented_flag(dk, dv):
    """The state updated in place (two CTAs write the two row halves of one
    state when Dv = 256), bitwise run-to-run determinism, and the segmented
    entry point (which runs the single pass at these dims) giving the same bits."""
    gdn = _gdn()
    d = to_dev(inputs.prefill_inputs(2, 200, 3, dk, dv, seed=31 + dk, s0_std=0.05))
    o1, S1 = gdn.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], segmented=False)
    o2, S2 = gdn.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], segmented=True)
    S_in = d["S0"].clone()
    o3, S3 = gdn.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], S_in, S_T=S_in)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(S1, S2)
    assert torch.equal(o3, o1) and torch.equal(S3, S1) and S3.data_ptr() == S_in.data_ptr()


def test_tensor_core_head_dims_many_chains_sampled():
    """128 x 256 at B4 H32 T1024 (256 CTAs, two per chain), checked on sampled chains."""
    gdn = _gdn()
    B, T, H, dk, dv = 4, 1024, 32, 128, 256
    d = inputs.prefill_inputs(B, T, H, dk, dv, seed=5, g_mean=2.0)
    dd = to_dev(d)
    o, S_T = gdn.prefill(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], None)
    torch.cuda.synchronize()
    chains = [0, 37, 127]
    ro, rS = oracle.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], None, chains=chains)
    o, S_T = o.cpu().numpy(), S_T.cpu().numpy()
    for c in chains:
        b, h = divmod(c, H)
        assert_parity(o[b, :, h], ro[b, :, h], f"o chain {c}")
        assert_parity(S_T[b, h], rS[b, h], f"S_T chain {c}")


def test_row_kernel_dims_reject_fused_options_on_gpu():
    """Dk = 256 (the row kernel) has no fused options; nor has decode outside
    64 x 64 and 128 x 128."""
    gdn = _gdn()
    d = to_dev(inputs.prefill_inputs(1, 16, 2, 256, 256, seed=22))
    with pytest.raises(gdn.GDNError) as e:
        gdn.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], qk_l2norm=True)
    assert e.value.code == gdn.GDN_ERR_UNSUPPORTED
    e2 = to_dev(inputs.prefill_inputs(2, 1, 2, 64, 128, seed=23, s0_std=0.02))
    with pytest.raises(gdn.GDNError) as e:
        gdn.decode_tokens(e2["q"], e2["k"], e2["v"], e2["g"], e2["beta"], e2["S0"].clone(), q_scale=0.5)
    assert e.value.code == gdn.GDN_ERR_UNSUPPORTED


TC_DIMS = [(64, 64), (64, 128), (128, 64), (128, 256)]


@pytest.mark.parametrize("chunk", [64, 16])
@pytest.mark.parametrize("dk,dv", TC_DIMS, ids=[f"{a}x{b}" for a, b in TC_DIMS])
def test_fused_options_tensor_core_head_dims(dk, dv, chunk):
    """q / k L2 normalisation and the q scale fused into the tensor-core kernel
    at the other head dims equal the oracle run on inputs normalised in fp64
    beforehand; bf16 o is the fp32 o rounded to nearest even, bit for bit, with
    the same end state.  T = 150 leaves a ragged last tile."""
    gdn = _gdn()
    d = inputs.prefill_inputs(2, 150, 3, dk, dv, seed=400 + dk + dv + chunk, s0_std=0.05)
    r = raw_qk(d, 401 + dk + dv)
    qs = dk ** -0.5
    dd = to_dev(d)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, S_T = gdn.prefill(r["q"].to(DEV), r["k"].to(DEV), dd["v"], dd["g"], dd["beta"], dd["S0"],
                         chunk=chunk, qk_l2norm=True, q_scale=qs, status=status)
    assert gdn.query_status(status) == 0
    ro, rS = oracle.prefill((r["q_n"] * qs).float(), r["k_n"].float(), d["v"], d["g"], d["beta"],
                            d["S0"])
    assert_parity(o.cpu().numpy(), ro, f"o (fused norm) {dk}x{dv}")
    assert_parity(S_T.cpu().numpy(), rS, f"S_T (fused norm) {dk}x{dv}")
    o16, S16 = gdn.prefill(r["q"].to(DEV), r["k"].to(DEV), dd["v"], dd["g"], dd["beta"], dd["S0"],
                           chunk=chunk, qk_l2norm=True, q_scale=qs, o_bf16=True, status=status)
    assert gdn.query_status(status) == 0
    assert o16.dtype == torch.bfloat16
    assert torch.equal(o16, o.to(torch.bfloat16))
    assert torch.equal(S16, S_T)


@pytest.mark.parametrize("dk,dv", TC_DIMS, ids=[f"{a}x{b}" for a, b in TC_DIMS])
def test_default_options_are_bitwise_the_plain_call_at_other_head_dims(dk, dv):
    """Default options through gdn_prefill_ex give bitwise the plain call's
    results (at these dims the plain call runs the kernel with the pre-steps
    compiled in, their factors exactly 1)."""
    import ctypes as ct
    gdn = _gdn()
    B, T, H = 2, 130, 3
    d = to_dev(inputs.prefill_inputs(B, T, H, dk, dv, seed=420 + dk + dv, s0_std=0.02))
    o1, S1 = gdn.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], segmented=False)
    o2 = torch.empty_like(o1)
    S2 = torch.empty_like(S1)
    opts = gdn.Options(ct.sizeof(gdn.Options), 0, 1.0, 0)
    rc = gdn.raw_prefill_ex(*[ct.c_void_p(t.data_ptr()) for t in (d["q"], d["k"], d["v"], d["g"],
                                                                    d["beta"], d["S0"], o2, S2)],
                            B, T, H, dk, dv, 64, None, ct.c_size_t(0), ct.byref(opts), None,
                            ct.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    assert rc == 0 and torch.equal(o1, o2) and torch.equal(S1, S2)


@pytest.mark.parametrize("T", [1, 3])
def test_fused_options_in_decode_64(T):
    """The 64 x 64 streaming decode with q / k normalised and q scaled in the
    kernel equals the oracle on fp64-normalised inputs; its bf16 o is the fp32
    o rounded, bit for bit."""
    gdn = _gdn()
    d = inputs.prefill_inputs(4, T, 8, 64, 64, seed=440 + T, s0_std=0.05)
    r = raw_qk(d, 441)
    qs = 0.5
    dd = to_dev(d)
    S = dd["S0"].clone()
    o = gdn.decode_tokens(r["q"].to(DEV), r["k"].to(DEV), dd["v"], dd["g"], dd["beta"], S,
                          qk_l2norm=True, q_scale=qs)
    torch.cuda.synchronize()
    ro, rS = oracle.prefill((r["q_n"] * qs).float(), r["k_n"].float(), d["v"], d["g"], d["beta"],
                            d["S0"])
    assert_parity(o.cpu().numpy(), ro, f"o T={T}")
    assert_parity(S.cpu().numpy(), rS, f"S T={T}")
    S2 = dd["S0"].clone()
    o16 = gdn.decode_tokens(r["q"].to(DEV), r["k"].to(DEV), dd["v"], dd["g"], dd["beta"], S2,
                            qk_l2norm=True, q_scale=qs, o_bf16=True)
    torch.cuda.synchronize()
    assert torch.equal(o16, o.to(torch.bfloat16)) and torch.equal(S2, S)


@pytest.mark.parametrize("T", [1, 3])
def test_kda_fused_options_in_decode_64(T):
    gdn = _gdn()
    d = inputs.kda_inputs(4, T, 8, 64, 64, seed=450 + T, s0_std=0.05)
    r = raw_qk(d, 451)
    qs = 0.5
    dd = to_dev(d)
    S = dd["S0"].clone()
    o = gdn.kda_decode(r["q"].to(DEV), r["k"].to(DEV), dd["v"], dd["g"], dd["beta"], S,
                       qk_l2norm=True, q_scale=qs)
    torch.cuda.synchronize()
    ro, rS = oracle.kda_prefill((r["q_n"] * qs).float(), r["k_n"].float(), d["v"], d["g"],
                                d["beta"], d["S0"])
    assert_parity(o.cpu().numpy(), ro, f"o T={T}")
    assert_parity(S.cpu().numpy(), rS, f"S T={T}")


def _packed(lengths, H, dk, dv, seed, s0_std=None):
    """Packed inputs of sequences of the given lengths at head dims dk x dv:
    per-sequence draws of the seeded generator, concatenated along tokens."""
    seqs = [inputs.prefill_inputs(1, L, H, dk, dv, seed=seed + i, s0_std=s0_std)
            for i, L in enumerate(lengths)]
    cat = lambda key: torch.cat([d[key][0] for d in seqs], 0)
    S0 = torch.cat([d["S0"] for d in seqs], 0) if s0_std else None
    cu = torch.tensor([0] + list(np.cumsum(lengths)), dtype=torch.int32)
    return seqs, dict(q=cat("q"), k=cat("k"), v=cat("v"), g=cat("g"), beta=cat("beta"), S0=S0, cu=cu)


VARLEN_DIMS = [(64, 64), (64, 128), (128, 64), (128, 256), (64, 256)]


@pytest.mark.parametrize("chunk", [64, 16])
@pytest.mark.parametrize("dk,dv", VARLEN_DIMS, ids=[f"{a}x{b}" for a, b in VARLEN_DIMS])
def test_varlen_packed_sequences_other_head_dims(dk, dv, chunk):
    """Packed sequences of mixed lengths (empty, 1 token, ragged, tile-aligned)
    at the tensor-core head dims, each against the oracle run on that sequence
    alone; an empty sequence's S_T is its S0."""
    lengths = [130, 0, 1, 64, 77]
    H = 2
    seqs, pk = _packed(lengths, H, dk, dv, seed=500 + dk + dv, s0_std=0.05)
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
        assert_parity(S_T[n], rS[0], f"S_T seq {n} (len {lengths[n]})")


@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 256), (64, 128)], ids=["64x64", "128x256", "64x128"])
def test_varlen_state_snapshots_other_head_dims(dk, dv):
    """Snapshots after every 64 tokens of each sequence equal the oracle's state
    on that prefix (a sequence of 128 tokens ends on a snapshot: its last one is
    its S_T); the outputs equal those of the call without snapshots."""
    lengths = [130, 64, 0, 128]
    H = 2
    seqs, pk = _packed(lengths, H, dk, dv, seed=530 + dk + dv, s0_std=0.05)
    gdn = _gdn()
    dd = to_dev(pk)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, S_T, snaps = gdn.prefill_varlen(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["cu"],
                                       dd["S0"], status=status, snap_every=64)
    assert gdn.query_status(status) == 0
    assert tuple(snaps.shape) == (sum(L // 64 for L in lengths), H, dv, dk)
    sn = snaps.cpu().numpy()
    slot = 0
    for n, d in enumerate(seqs):
        for j in range(1, lengths[n] // 64 + 1):
            t = 64 * j
            cut = lambda x: x[:, :t]
            _, rS = oracle.prefill(cut(d["q"]), cut(d["k"]), cut(d["v"]), cut(d["g"]), cut(d["beta"]),
                                   d["S0"])
            assert_parity(sn[slot], rS[0], f"snapshot {j} of seq {n} (t={t})")
            slot += 1
    o2, S2 = gdn.prefill_varlen(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["cu"], dd["S0"])
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(S_T, S2)


@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 256)], ids=["64x64", "128x256"])
def test_varlen_snapshot_bounds_other_head_dims(dk, dv):
    """Snapshot slots at other head dims stay inside the buffer: malformed
    offsets (a sequence ending before it starts) leave the slots in front of the
    buffer untouched, and a buffer one slot short leaves the slot after it
    untouched; both report GDN_ERR_SHAPE."""
    H, T = 2, 200
    d = inputs.prefill_inputs(1, T, H, dk, dv, seed=560 + dk + dv)
    gdn = _gdn()
    flat = lambda x: x[0].contiguous().to(DEV)
    args = [flat(d[key]) for key in ("q", "k", "v", "g", "beta")]
    guard = 2
    buf = torch.full((guard + 3 + guard, H, dv, dk), 7.0, dtype=torch.float32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    bad = torch.tensor([100, 0, 200], dtype=torch.int32, device=DEV)
    gdn.prefill_varlen(*args, bad, status=status, snap_every=64, snaps=buf[guard:guard + 3])
    assert gdn.query_status(status) == gdn.GDN_ERR_SHAPE
    assert torch.all(buf[:guard] == 7.0) and torch.all(buf[guard + 3:] == 7.0)
    # 200 tokens need 3 slots; give 2
    status.zero_()
    ok = torch.tensor([0, 200], dtype=torch.int32, device=DEV)
    gdn.prefill_varlen(*args, ok, status=status, snap_every=64, snaps=buf[guard:guard + 2])
    assert gdn.query_status(status) == gdn.GDN_ERR_SHAPE
    assert torch.all(buf[:guard] == 7.0) and torch.all(buf[guard + 2:] == 7.0)


@pytest.mark.parametrize("dv", [64, 256])
def test_kda_tensor_core_prefill_other_value_dims(dv):
    """The per-channel-gate prefill at Dk = 128 with Dv = 64 (lanes 64..127 of
    the state stay zero) or Dv = 256 (two CTAs per chain) on the chunked
    tensor-core kernel: whole and ragged 32-token tiles, carried state, strong
    and weak decays, with and without the fused q/k norm and q scale."""
    gdn = _gdn()
    for T, g_mean, norm in ((100, 0.0, False), (33, 2.0, True), (64, -3.0, False)):
        d = inputs.kda_inputs(2, T, 3, 128, dv, seed=600 + dv + T, g_mean=g_mean, s0_std=0.05)
        r = raw_qk(d, 601 + T) if norm else {"q": d["q"], "k": d["k"], "q_n": d["q"].double(),
                                               "k_n": d["k"].double()}
        qs = 128 ** -0.5 if norm else 1.0
        dd = to_dev(d)
        status = torch.zeros(1, dtype=torch.int32, device=DEV)
        o, S_T = gdn.kda_prefill(r["q"].to(DEV), r["k"].to(DEV), dd["v"], dd["g"], dd["beta"], dd["S0"],
                                 status=status, qk_l2norm=norm, q_scale=qs)
        assert gdn.query_status(status) == 0
        ro, rS = oracle.kda_prefill((r["q_n"] * qs).float(), r["k_n"].float(), d["v"], d["g"], d["beta"],
                                    d["S0"])
        assert_parity(o.cpu().numpy(), ro, f"o kda 128x{dv} T={T}")
        assert_parity(S_T.cpu().numpy(), rS, f"S_T kda 128x{dv} T={T}")
    # in place and deterministic
    S = dd["S0"].clone()
    o1, _ = gdn.kda_prefill(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], S, S_T=S)
    o2, S2 = gdn.kda_prefill(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["S0"])
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(S, S2)
