"""GPU parity of the per-channel-gate (KDA) kernels, through the C ABI, against
the fp64 KDA oracle on the same seeded inputs.

Prefill at Dk = Dv = 128 runs the chunked tensor-core kernel (32-token
chunks, every derived operand as a bf16 hi/lo pair); decode at Dk = Dv = 128
or 64 runs the streaming decode kernel (the per-column decay applied to each
state row in registers); the other head dims run the row kernel, which walks
the tokens in fp32 in the order of the recurrence.  The same contract as the scalar-gate path applies (relative
Frobenius <= 2e-3, max-abs <= 1e-2 x RMS on o and S_T), and the tighter 1e-4
design margin is asserted too.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_linear_20_b200 import inputs
from tests.test_gpu_parity import DEV, assert_parity, to_dev

pytestmark = pytest.mark.gpu


def _gdn():
    from gated_deltanet_linear_20_b200 import gdn
    return gdn


def _run(d, **kw):
    dd = to_dev(d)
    o, S_T = _gdn().kda_prefill(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["S0"], **kw)
    torch.cuda.synchronize()
    return o.cpu().numpy(), S_T.cpu().numpy()


def _check(d, what):
    o, S_T = _run(d)
    ro, rS = oracle.kda_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    assert_parity(o, ro, f"o {what}")
    assert_parity(S_T, rS, f"S_T {what}")


def test_kda_tiny_b1_h2_t64():
    _check(inputs.kda_inputs(1, 64, 2, seed=0), "B1 H2 T64")


@pytest.mark.parametrize("T", [1, 11, 12, 13, 100])
@pytest.mark.parametrize("BH", [(1, 4), (3, 16), (8, 16)], ids=["16rows_4heads", "16rows", "32rows"])
def test_kda_ragged_lengths_all_cta_shapes(T, BH):
    """On 148 SMs, B*H = 4 and 48 run 16 rows per CTA, 128 runs 32 rows per
    CTA; T covers the direct single-token path, partial and exact 12-token
    chunks (a warp converts up to 3 tokens of a chunk)."""
    B, H = BH
    _check(inputs.kda_inputs(B, T, H, seed=T, s0_std=0.05), f"B{B} H{H} T{T}")


def test_kda_b1_h16_t512():
    _check(inputs.kda_inputs(1, 512, 16, seed=0), "B1 H16 T512")


def test_kda_long_memory_t4096_carried_state():
    """Slow decays (g = logsigmoid(N(2, 1)) per channel) over 4096 tokens from a
    carried state: rounding has the longest time to accumulate."""
    _check(inputs.kda_inputs(1, 4096, 4, seed=3, g_mean=2.0, s0_std=0.02), "B1 H4 T4096")


def test_kda_sampled_chains_b4_h32_t2048():
    """A large launch (128 chains, 32 rows per CTA) checked on three sampled
    chains, each run through the oracle on its own slice of the inputs."""
    d = inputs.kda_inputs(4, 2048, 32, seed=5, g_mean=2.0, device=DEV)
    gdn = _gdn()
    o, S_T = gdn.kda_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], None)
    torch.cuda.synchronize()
    for b, h in ((0, 0), (2, 17), (3, 31)):
        sl = lambda x: x[b:b + 1, :, h:h + 1].cpu()
        ro, rS = oracle.kda_prefill(sl(d["q"]), sl(d["k"]), sl(d["v"]), sl(d["g"]), sl(d["beta"]))
        assert_parity(o[b:b + 1, :, h:h + 1].cpu().numpy(), ro, f"o chain ({b},{h})")
        assert_parity(S_T[b:b + 1, h:h + 1].cpu().numpy(), rS, f"S_T chain ({b},{h})")


def test_kda_decode_b64_h16_steps():
    """Decode: 8 single-token calls on 64 x 16 heads, the state in place,
    against the oracle run over the 8 tokens at once; then a 4-token call."""
    d = inputs.kda_inputs(64, 12, 16, seed=7, s0_std=0.02)
    dd = to_dev(d)
    gdn = _gdn()
    S = dd["S0"].clone()
    outs = []
    step = lambda sl: [dd[key][:, sl].contiguous() for key in ("q", "k", "v", "g", "beta")]
    for t in range(8):
        outs.append(gdn.kda_decode(*step(t), S))
    o4 = gdn.kda_decode(*step(slice(8, 12)), S)
    torch.cuda.synchronize()
    ro, rS = oracle.kda_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    o = torch.cat([torch.stack(outs, 1), o4], 1).cpu().numpy()
    assert_parity(o, ro, "o decode")
    assert_parity(S.cpu().numpy(), rS, "S decode")


@pytest.mark.parametrize("D", [128, 64])
@pytest.mark.parametrize("g_mean,label", [(-3.0, "strong"), (4.0, "weak"), (None, "growing")])
def test_kda_decode_decay_strengths(D, g_mean, label):
    """Decode at 128 x 128 and 64 x 64 with per-channel decays of several
    strengths (and positive log decays, which grow the state): 3 single-token
    steps, a 2-token and a 5-token burst, against the oracle over the 10
    tokens."""
    d = inputs.kda_inputs(8, 10, 5, D, D, seed=40 + D, s0_std=0.05,
                          g_mean=g_mean if g_mean is not None else -3.0)
    if g_mean is None:
        d["g"] = (d["g"].abs() * 0.05).contiguous()
    dd = to_dev(d)
    gdn = _gdn()
    S = dd["S0"].clone()
    step = lambda sl: [dd[key][:, sl].contiguous() for key in ("q", "k", "v", "g", "beta")]
    outs = [gdn.kda_decode(*step(t), S).unsqueeze(1) for t in range(3)]
    outs.append(gdn.kda_decode(*step(slice(3, 5)), S))
    outs.append(gdn.kda_decode(*step(slice(5, 10)), S))
    torch.cuda.synchronize()
    ro, rS = oracle.kda_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    assert_parity(torch.cat(outs, 1).cpu().numpy(), ro, f"o kda decode {D} {label}")
    assert_parity(S.cpu().numpy(), rS, f"S kda decode {D} {label}")


def test_kda_decode_64_b64_h16_steps():
    """The 64 x 64 decode at 64 x 16 heads: 6 single-token steps and a 2-token
    burst on every head, against the oracle."""
    d = inputs.kda_inputs(64, 8, 16, 64, 64, seed=17, s0_std=0.02)
    dd = to_dev(d)
    gdn = _gdn()
    S = dd["S0"].clone()
    step = lambda sl: [dd[key][:, sl].contiguous() for key in ("q", "k", "v", "g", "beta")]
    outs = [gdn.kda_decode(*step(t), S).unsqueeze(1) for t in range(6)]
    outs.append(gdn.kda_decode(*step(slice(6, 8)), S))
    torch.cuda.synchronize()
    ro, rS = oracle.kda_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    assert_parity(torch.cat(outs, 1).cpu().numpy(), ro, "o kda decode 64x64")
    assert_parity(S.cpu().numpy(), rS, "S kda decode 64x64")


def test_kda_in_place_zero_length_and_determinism():
    gdn = _gdn()
    d = to_dev(inputs.kda_inputs(2, 40, 3, seed=9, s0_std=0.05))
    o1, S1 = gdn.kda_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    o2, S2 = gdn.kda_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    S_in = d["S0"].clone()
    o3, S3 = gdn.kda_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], S_in, S_T=S_in)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(S1, S2), "not bitwise run-to-run"
    assert S3.data_ptr() == S_in.data_ptr()
    assert torch.equal(o3, o1) and torch.equal(S3, S1), "in place differs from out of place"
    # T = 0: S_T is S0, or zeros without S0
    e = {k: (v[:, :0].contiguous() if k != "S0" else v) for k, v in d.items()}
    _, Z = gdn.kda_prefill(e["q"], e["k"], e["v"], e["g"], e["beta"], d["S0"])
    _, Z0 = gdn.kda_prefill(e["q"], e["k"], e["v"], e["g"], e["beta"], None,
                            S_T=torch.full_like(d["S0"], 7.0))
    torch.cuda.synchronize()
    assert torch.equal(Z, d["S0"]) and not Z0.any()


def test_kda_equal_gates_match_the_scalar_gate_oracle():
    """A gate equal on every key channel is the scalar gated delta rule: the
    KDA kernel on such inputs agrees with the scalar-gate oracle."""
    d = inputs.prefill_inputs(1, 200, 4, seed=11, s0_std=0.05)
    kd = dict(d)
    kd["g"] = d["g"][..., None].expand(*d["g"].shape, 128).contiguous()
    o, S_T = _run(kd)
    ro, rS = oracle.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    assert_parity(o, ro, "o equal gates")
    assert_parity(S_T, rS, "S_T equal gates")


def _check_status(d, what):
    gdn = _gdn()
    dd = to_dev(d)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, S_T = gdn.kda_prefill(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["S0"], status=status)
    assert gdn.query_status(status) == 0, "a device-side wait timed out"
    ro, rS = oracle.kda_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    assert_parity(o.cpu().numpy(), ro, f"o {what}")
    assert_parity(S_T.cpu().numpy(), rS, f"S_T {what}")


@pytest.mark.parametrize("T", [31, 32, 33, 65, 257])
def test_kda_chunk_edges(T):
    """Lengths around the 32-token chunk: one short chunk, exactly one, one
    token into the second, and longer ragged runs; S0 carried in."""
    _check_status(inputs.kda_inputs(2, T, 3, seed=40 + T, s0_std=0.05), f"B2 H3 T{T}")


@pytest.mark.parametrize("g_mean", [-3.0, -1.0, 4.0], ids=["strong", "medium", "weak"])
def test_kda_decay_strengths(g_mean):
    """Per-channel gates logsigmoid(N(g_mean, 1)): mean log-decay about -3 per
    token (a channel's decay over a 32-token chunk reaches ~e^-100, far below
    the fp32 range, so in-chunk factors underflow), about -1.3, and about
    -0.02 (long memory)."""
    d = inputs.kda_inputs(1, 300, 4, seed=50, g_mean=g_mean, s0_std=0.05)
    if g_mean == -3.0:
        g = d["g"].numpy().astype(np.float64)
        assert g[0, :32].sum(0).min() < -87.0  # the premise: underflow inside one chunk
    _check_status(d, f"g_mean {g_mean}")


def test_kda_sampled_chains_b4_h32_t8192():
    """The benchmark shape (128 chains x 8192 tokens, long memory), three
    chains checked against the oracle on their own slices."""
    d = inputs.kda_inputs(4, 8192, 32, seed=6, g_mean=2.0, device=DEV)
    gdn = _gdn()
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, S_T = gdn.kda_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], None, status=status)
    assert gdn.query_status(status) == 0
    for b, h in ((0, 0), (1, 9), (3, 31)):
        sl = lambda x: x[b:b + 1, :, h:h + 1].cpu()
        ro, rS = oracle.kda_prefill(sl(d["q"]), sl(d["k"]), sl(d["v"]), sl(d["g"]), sl(d["beta"]))
        assert_parity(o[b:b + 1, :, h:h + 1].cpu().numpy(), ro, f"o chain ({b},{h})")
        assert_parity(S_T[b:b + 1, h:h + 1].cpu().numpy(), rS, f"S_T chain ({b},{h})")


def test_kda_prefill_then_decode_continue_one_state():
    """A prefill (tensor cores) followed by decode steps (row kernel) on the
    state it leaves: the two kernels must agree on the state's layout and
    meaning; checked against the oracle over all tokens."""
    d = inputs.kda_inputs(2, 70, 3, seed=60, s0_std=0.05)
    dd = to_dev(d)
    gdn = _gdn()
    pre = {k: v[:, :64].contiguous() for k, v in dd.items() if k != "S0"}
    o1, S = gdn.kda_prefill(pre["q"], pre["k"], pre["v"], pre["g"], pre["beta"], dd["S0"])
    o2 = gdn.kda_decode(*[dd[k][:, 64:].contiguous() for k in ("q", "k", "v", "g", "beta")], S)
    torch.cuda.synchronize()
    ro, rS = oracle.kda_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    assert_parity(torch.cat([o1, o2], 1).cpu().numpy(), ro, "o prefill + decode")
    assert_parity(S.cpu().numpy(), rS, "S prefill + decode")


def _raw_qk(d, seed):
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
        out[key + "_n"] = r64 / torch.sqrt((r64 * r64).sum(-1, keepdim=True) + 1e-6)
    return out


@pytest.mark.parametrize("norm,qs", [(True, 128 ** -0.5), (False, 0.5)], ids=["l2norm+scale", "scale"])
def test_kda_fused_qk_norm_and_q_scale(norm, qs):
    """The per-channel-gate prefill with q / k normalised and q scaled inside
    the kernel (gdn_kda_prefill_ex) equals the oracle run on inputs normalised
    in fp64 beforehand; T = 300 covers whole and ragged 32-token tiles."""
    d = inputs.kda_inputs(2, 300, 3, seed=151, s0_std=0.05)
    r = _raw_qk(d, 152) if norm else {"q": d["q"], "k": d["k"], "q_n": d["q"].double(), "k_n": d["k"].double()}
    dd = to_dev(d)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    gdn = _gdn()
    o, S_T = gdn.kda_prefill(r["q"].to(DEV), r["k"].to(DEV), dd["v"], dd["g"], dd["beta"], dd["S0"],
                             status=status, qk_l2norm=norm, q_scale=qs)
    assert gdn.query_status(status) == 0
    ro, rS = oracle.kda_prefill((r["q_n"] * qs).float(), r["k_n"].float(), d["v"], d["g"], d["beta"], d["S0"])
    assert_parity(o.cpu().numpy(), ro, "o (fused norm)")
    assert_parity(S_T.cpu().numpy(), rS, "S_T (fused norm)")


@pytest.mark.parametrize("T", [1, 3])
def test_kda_fused_qk_norm_in_decode(T):
    d = inputs.kda_inputs(4, T, 8, seed=160 + T, s0_std=0.05)
    r = _raw_qk(d, 161)
    qs = 0.5
    gdn = _gdn()
    dd = to_dev(d)
    S = dd["S0"].clone()
    o = gdn.kda_decode(r["q"].to(DEV), r["k"].to(DEV), dd["v"], dd["g"], dd["beta"], S,
                       qk_l2norm=True, q_scale=qs)
    torch.cuda.synchronize()
    ro, rS = oracle.kda_prefill((r["q_n"] * qs).float(), r["k_n"].float(), d["v"], d["g"], d["beta"], d["S0"])
    assert_parity(o.cpu().numpy(), ro, f"o T={T}")
    assert_parity(S.cpu().numpy(), rS, f"S T={T}")


def test_kda_default_options_are_bitwise_the_plain_call():
    """Default options through gdn_kda_prefill_ex run the same kernel as the
    plain call: bitwise the same results."""
    import ctypes as ct
    gdn = _gdn()
    d = to_dev(inputs.kda_inputs(2, 100, 3, seed=171, s0_std=0.02))
    o1, S1 = gdn.kda_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    o2 = torch.empty_like(o1)
    S2 = torch.empty_like(S1)
    opts = gdn.Options(ct.sizeof(gdn.Options), 0, 1.0, 0)
    rc = gdn.raw_kda_prefill_ex(*[ct.c_void_p(t.data_ptr()) for t in (d["q"], d["k"], d["v"], d["g"],
                                                                       d["beta"], d["S0"], o2, S2)],
                                2, 100, 3, 128, 128, ct.byref(opts), None,
                                ct.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


@pytest.mark.parametrize("T", [8, 33])
def test_kda_decode_long_bursts(T):
    """Per-channel-gate decode bursts of T tokens in one call (the state read
    and written once) against the oracle, o at every token and the end state."""
    d = inputs.kda_inputs(16, T, 4, seed=170 + T, s0_std=0.05, g_mean=-1.0)
    dd = to_dev(d)
    gdn = _gdn()
    S = dd["S0"].clone()
    o = gdn.kda_decode(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], S)
    torch.cuda.synchronize()
    ro, rS = oracle.kda_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    assert_parity(o.cpu().numpy(), ro, f"o kda burst T={T}")
    assert_parity(S.cpu().numpy(), rS, f"S kda burst T={T}")



@pytest.mark.parametrize("dv", [128, 64, 256])
def test_kda_bf16_o_is_the_fp32_o_rounded(dv):
    """o_bf16 in the per-channel-gate prefill stores the fp32 call's o rounded
    to nearest even, bit for bit, with an identical end state (T = 100: whole
    and ragged 32-token tiles); with the fused norm too at 128 x 128."""
    gdn = _gdn()
    d = to_dev(inputs.kda_inputs(2, 100, 3, 128, dv, seed=180 + dv, s0_std=0.05))
    for kw in ({}, dict(qk_l2norm=True, q_scale=0.25)) if dv == 128 else ({},):
        o32, S32 = gdn.kda_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], **kw)
        o16, S16 = gdn.kda_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], o_bf16=True, **kw)
        torch.cuda.synchronize()
        assert o16.dtype == torch.bfloat16
        assert torch.equal(o16, o32.to(torch.bfloat16)), f"dv={dv} {kw}"
        assert torch.equal(S16, S32), f"dv={dv} {kw}"


@pytest.mark.parametrize("D,T", [(128, 1), (128, 5), (64, 1), (64, 3)])
def test_kda_bf16_o_in_decode(D, T):
    gdn = _gdn()
    d = to_dev(inputs.kda_inputs(8, T, 4, D, D, seed=190 + D + T, s0_std=0.05))
    S32 = d["S0"].clone()
    S16 = d["S0"].clone()
    args = [d[key] for key in ("q", "k", "v", "g", "beta")]
    o32 = gdn.kda_decode(*args, S32)
    o16 = gdn.kda_decode(*args, S16, o_bf16=True)
    torch.cuda.synchronize()
    assert o16.dtype == torch.bfloat16
    assert torch.equal(o16, o32.to(torch.bfloat16)) and torch.equal(S16, S32)


def _kda_packed(lengths, H, dv, seed, s0_std=None):
    """Packed per-channel-gate inputs: per-sequence draws of the seeded
    generator, concatenated along tokens."""
    seqs = [inputs.kda_inputs(1, L, H, Dv=dv, seed=seed + i, s0_std=s0_std)
            for i, L in enumerate(lengths)]
    cat = lambda key: torch.cat([d[key][0] for d in seqs], 0)
    S0 = torch.cat([d["S0"] for d in seqs], 0) if s0_std else None
    cu = torch.tensor([0] + list(np.cumsum(lengths)), dtype=torch.int32)
    return seqs, dict(q=cat("q"), k=cat("k"), v=cat("v"), g=cat("g"), beta=cat("beta"), S0=S0, cu=cu)


@pytest.mark.parametrize("dv,s0", [(128, None), (128, 0.05), (64, 0.05), (256, 0.05)],
                         ids=["128_zero_state", "128", "64", "256"])
def test_kda_varlen_packed_sequences(dv, s0):
    """Packed sequences of mixed lengths (empty, 1 token, ragged, exact 32-token
    tiles; a ragged sequence last, ending at the end of the packed arrays), each
    against the oracle run on that sequence alone; an empty sequence's S_T is
    its S0 (or zeros)."""
    lengths = [130, 0, 1, 32, 77, 33, 31, 45]
    H = 2
    seqs, pk = _kda_packed(lengths, H, dv, seed=700 + dv, s0_std=s0)
    gdn = _gdn()
    dd = to_dev(pk)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, S_T = gdn.kda_prefill_varlen(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["cu"],
                                    dd["S0"], status=status)
    assert gdn.query_status(status) == 0
    o, S_T = o.cpu().numpy(), S_T.cpu().numpy()
    cu = pk["cu"].numpy()
    for n, d in enumerate(seqs):
        if lengths[n]:
            ro, rS = oracle.kda_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
            assert_parity(o[cu[n]:cu[n + 1]], ro[0], f"o seq {n} (len {lengths[n]})")
            assert_parity(S_T[n], rS[0], f"S_T seq {n} (len {lengths[n]})")
        elif s0:
            np.testing.assert_array_equal(S_T[n], d["S0"][0].numpy())
        else:
            np.testing.assert_array_equal(S_T[n], 0.0)


def test_kda_varlen_equal_lengths_match_the_dense_call():
    """Equal lengths packed = the dense [B][T][H] call, bitwise: the tokens of
    the next sequence in a last tile enter as padding (g = beta = 0), which
    contributes exact zeros, as the zero fill past T does in the dense call."""
    B, T, H = 3, 150, 4
    d = to_dev(inputs.kda_inputs(B, T, H, seed=8, s0_std=0.05))
    gdn = _gdn()
    o1, S1 = gdn.kda_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    cu = torch.arange(0, (B + 1) * T, T, dtype=torch.int32, device=DEV)
    flat = lambda x: x.reshape(B * T, *x.shape[2:]).contiguous()
    o2, S2 = gdn.kda_prefill_varlen(flat(d["q"]), flat(d["k"]), flat(d["v"]), flat(d["g"]),
                                    flat(d["beta"]), cu, d["S0"])
    torch.cuda.synchronize()
    assert torch.equal(o1.reshape(B * T, H, 128), o2) and torch.equal(S1, S2)


def test_kda_varlen_bad_offsets_are_reported_on_the_device():
    _, pk = _kda_packed([40, 40], 2, 128, seed=3)
    gdn = _gdn()
    dd = to_dev(pk)
    bad = torch.tensor([0, 50, 30], dtype=torch.int32, device=DEV)  # out of order
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    gdn.kda_prefill_varlen(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], bad, status=status)
    assert gdn.query_status(status) == gdn.GDN_ERR_SHAPE


def test_kda_varlen_all_sequences_empty_copy_the_state():
    H = 3
    S0 = torch.randn(2, H, 128, 128, device=DEV)
    e = lambda *s, dt=torch.bfloat16: torch.empty(*s, dtype=dt, device=DEV)
    cu = torch.zeros(3, dtype=torch.int32, device=DEV)
    gdn = _gdn()
    o, S_T = gdn.kda_prefill_varlen(e(0, H, 128), e(0, H, 128), e(0, H, 128),
                                    e(0, H, 128, dt=torch.float32), e(0, H, dt=torch.float32), cu, S0)
    torch.cuda.synchronize()
    assert o.shape == (0, H, 128) and torch.equal(S_T, S0)


@pytest.mark.parametrize("dv,snap_every", [(128, 32), (128, 64), (256, 96), (64, 32)],
                         ids=["128_every32", "128_every64", "256_every96", "64_every32"])
def test_kda_varlen_state_snapshots(dv, snap_every):
    """Snapshots after every snap_every tokens of each sequence equal the oracle's
    state on that prefix (a sequence ending on a boundary: its last snapshot is
    S_T); the outputs are unchanged by taking them."""
    lengths = [200, 64, 0, 129, 96, 31]
    H = 2
    seqs, pk = _kda_packed(lengths, H, dv, seed=760 + dv + snap_every, s0_std=0.05)
    gdn = _gdn()
    dd = to_dev(pk)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, S_T, snaps = gdn.kda_prefill_varlen(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["cu"],
                                           dd["S0"], status=status, snap_every=snap_every)
    assert gdn.query_status(status) == 0
    assert snaps.shape[0] == sum(L // snap_every for L in lengths)
    snaps = snaps.cpu().numpy()
    slot = 0
    for n, d in enumerate(seqs):
        for j in range(1, lengths[n] // snap_every + 1):
            t = j * snap_every
            cut = lambda x: x[:, :t]
            _, rS = oracle.kda_prefill(cut(d["q"]), cut(d["k"]), cut(d["v"]), cut(d["g"]),
                                       cut(d["beta"]), d["S0"])
            assert_parity(snaps[slot], rS[0], f"snapshot {j} of seq {n} (t={t})")
            slot += 1
    o2, S2 = gdn.kda_prefill_varlen(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["cu"], dd["S0"])
    torch.cuda.synchronize()
    assert torch.equal(o.cpu(), o2.cpu()) and torch.equal(S_T.cpu(), S2.cpu())


@pytest.mark.parametrize("dv", [128, 256])
def test_kda_varlen_snapshot_bounds(dv):
    """Snapshot slots stay inside the buffer: malformed offsets (a sequence
    ending before it starts) leave the slots in front of the buffer untouched,
    and a buffer one slot short leaves the slot after it untouched; both report
    GDN_ERR_SHAPE."""
    H, T = 2, 200
    d = inputs.kda_inputs(1, T, H, Dv=dv, seed=780 + dv)
    gdn = _gdn()
    flat = lambda x: x[0].contiguous().to(DEV)
    args = [flat(d[key]) for key in ("q", "k", "v", "g", "beta")]
    guard = 2
    buf = torch.full((guard + 3 + guard, H, dv, 128), 7.0, dtype=torch.float32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    bad = torch.tensor([100, 0, 200], dtype=torch.int32, device=DEV)
    gdn.kda_prefill_varlen(*args, bad, status=status, snap_every=64, snaps=buf[guard:guard + 3])
    assert gdn.query_status(status) == gdn.GDN_ERR_SHAPE
    assert torch.all(buf[:guard] == 7.0) and torch.all(buf[guard + 3:] == 7.0)
    # 200 tokens need 3 slots of 64; give 2
    status.zero_()
    ok = torch.tensor([0, 200], dtype=torch.int32, device=DEV)
    gdn.kda_prefill_varlen(*args, ok, status=status, snap_every=64, snaps=buf[guard:guard + 2])
    assert gdn.query_status(status) == gdn.GDN_ERR_SHAPE
    assert torch.all(buf[:guard] == 7.0) and torch.all(buf[guard + 2:] == 7.0)


def test_kda_varlen_benchmark_workload_sampled_chains():
    """The packed benchmark workload (32 sequences of seeded uniform 64..2048
    tokens, 16 heads), drawn on the device as the benchmark draws it; four
    (sequence, head) chains, the longest sequence among them, checked against
    the oracle on their own slices."""
    rng = np.random.default_rng(4000)
    lens = rng.integers(64, 2049, size=32)
    seqs = [inputs.kda_inputs(1, int(L), 16, seed=5200 + i, device=DEV) for i, L in enumerate(lens)]
    pk = {key: torch.cat([d[key][0] for d in seqs], 0) for key in ("q", "k", "v", "g", "beta")}
    del seqs
    cu_h = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    cu = torch.from_numpy(cu_h).to(DEV)
    gdn = _gdn()
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, S_T = gdn.kda_prefill_varlen(pk["q"], pk["k"], pk["v"], pk["g"], pk["beta"], cu, status=status)
    assert gdn.query_status(status) == 0
    longest = int(np.argmax(lens))
    for n, h in ((0, 0), (longest, 7), (17, 15), (31, 3)):
        t0, t1 = int(cu_h[n]), int(cu_h[n + 1])
        sl = lambda x: x[t0:t1, h:h + 1].unsqueeze(0).cpu()
        ro, rS = oracle.kda_prefill(sl(pk["q"]), sl(pk["k"]), sl(pk["v"]), sl(pk["g"]), sl(pk["beta"]))
        assert_parity(o[t0:t1, h:h + 1].unsqueeze(0).cpu().numpy(), ro, f"o seq {n} head {h}")
        assert_parity(S_T[n:n + 1, h:h + 1].cpu().numpy(), rS, f"S_T seq {n} head {h}")


@pytest.mark.parametrize("dv", [128, 64, 256])
def test_kda_varlen_fused_qk_norm_and_q_scale(dv):
    """Packed per-channel-gate sequences with q / k normalised and q scaled in
    the kernel (gdn_kda_prefill_varlen_ex) equal the oracle run per sequence on
    inputs normalised in fp64 beforehand; snapshots are taken on the way."""
    lengths = [130, 0, 1, 64, 77]
    H, qs = 2, 0.5
    seqs, pk = _kda_packed(lengths, H, dv, seed=800 + dv, s0_std=0.05)
    r = _raw_qk(pk, 801 + dv)
    dd = to_dev(pk)
    gdn = _gdn()
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, S_T, snaps = gdn.kda_prefill_varlen(r["q"].to(DEV), r["k"].to(DEV), dd["v"], dd["g"], dd["beta"],
                                           dd["cu"], dd["S0"], status=status, snap_every=64,
                                           qk_l2norm=True, q_scale=qs)
    assert gdn.query_status(status) == 0
    o, S_T, snaps = o.cpu().numpy(), S_T.cpu().numpy(), snaps.cpu().numpy()
    cu = pk["cu"].numpy()
    slot = 0
    for n, d in enumerate(seqs):
        t0, t1 = int(cu[n]), int(cu[n + 1])
        sl = lambda x, t=t1: x[t0:t].unsqueeze(0)
        if lengths[n]:
            ro, rS = oracle.kda_prefill((sl(r["q_n"]) * qs).float(), sl(r["k_n"]).float(), d["v"], d["g"],
                                        d["beta"], d["S0"])
            assert_parity(o[t0:t1], ro[0], f"o seq {n} (fused norm)")
            assert_parity(S_T[n], rS[0], f"S_T seq {n} (fused norm)")
        for j in range(1, lengths[n] // 64 + 1):
            te = t0 + 64 * j
            _, rS = oracle.kda_prefill((sl(r["q_n"], te) * qs).float(), sl(r["k_n"], te).float(),
                                       d["v"][:, :64 * j], d["g"][:, :64 * j], d["beta"][:, :64 * j], d["S0"])
            assert_parity(snaps[slot], rS[0], f"snapshot {j} of seq {n} (fused norm)")
            slot += 1
    assert slot == snaps.shape[0]


@pytest.mark.parametrize("dk,dv,chunk", [(128, 128, 64), (128, 128, 16), (64, 64, 64), (128, 256, 64)],
                         ids=["128x128_c64", "128x128_c16", "64x64", "128x256"])
def test_scalar_varlen_fused_qk_norm_and_q_scale(dk, dv, chunk):
    """Packed scalar-gate sequences with q / k normalised and q scaled in the
    kernel (gdn_prefill_varlen_ex) equal the oracle run per sequence on inputs
    normalised in fp64 beforehand."""
    lengths = [130, 0, 1, 64, 77]
    H, qs = 2, 0.5
    seqs = [inputs.prefill_inputs(1, L, H, dk, dv, seed=820 + i, s0_std=0.05)
            for i, L in enumerate(lengths)]
    cat = lambda key: torch.cat([d[key][0] for d in seqs], 0)
    pk = dict(q=cat("q"), k=cat("k"), v=cat("v"), g=cat("g"), beta=cat("beta"),
              S0=torch.cat([d["S0"] for d in seqs], 0),
              cu=torch.tensor([0] + list(np.cumsum(lengths)), dtype=torch.int32))
    r = _raw_qk(pk, 830 + dk + dv)
    dd = to_dev(pk)
    gdn = _gdn()
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, S_T = gdn.prefill_varlen(r["q"].to(DEV), r["k"].to(DEV), dd["v"], dd["g"], dd["beta"], dd["cu"],
                                dd["S0"], chunk=chunk, status=status, qk_l2norm=True, q_scale=qs)
    assert gdn.query_status(status) == 0
    o, S_T = o.cpu().numpy(), S_T.cpu().numpy()
    cu = pk["cu"].numpy()
    for n, d in enumerate(seqs):
        t0, t1 = int(cu[n]), int(cu[n + 1])
        if not lengths[n]:
            np.testing.assert_array_equal(S_T[n], d["S0"][0].numpy())
            continue
        sl = lambda x: x[t0:t1].unsqueeze(0)
        ro, rS = oracle.prefill((sl(r["q_n"]) * qs).float(), sl(r["k_n"]).float(), d["v"], d["g"],
                                d["beta"], d["S0"])
        assert_parity(o[t0:t1], ro[0], f"o seq {n} (fused norm)")
        assert_parity(S_T[n], rS[0], f"S_T seq {n} (fused norm)")


@pytest.mark.parametrize("gate,dims", [("kda", (128, 128)), ("kda", (128, 256)), ("kda", (128, 64)),
                                       ("scalar", (128, 128)), ("scalar", (64, 64)),
                                       ("scalar", (128, 256))],
                         ids=["kda_128", "kda_256", "kda_64", "scalar_128x128", "scalar_64x64",
                              "scalar_128x256"])
def test_varlen_bf16_o_is_the_fp32_o_rounded(gate, dims):
    """Packed sequences with bf16 o (the ragged last tile of each sequence
    copied out as bf16 rows) give the fp32 call's o rounded to nearest even,
    bit for bit, and the same S_T and snapshots."""
    dk, dv = dims
    lengths = [130, 0, 1, 64, 77, 33]
    H = 2
    if gate == "kda":
        seqs, pk = _kda_packed(lengths, H, dv, seed=900 + dv, s0_std=0.05)
        call, every = _gdn().kda_prefill_varlen, 64
    else:
        seqs = [inputs.prefill_inputs(1, L, H, dk, dv, seed=910 + i, s0_std=0.05)
                for i, L in enumerate(lengths)]
        cat = lambda key: torch.cat([d[key][0] for d in seqs], 0)
        pk = dict(q=cat("q"), k=cat("k"), v=cat("v"), g=cat("g"), beta=cat("beta"),
                  S0=torch.cat([d["S0"] for d in seqs], 0),
                  cu=torch.tensor([0] + list(np.cumsum(lengths)), dtype=torch.int32))
        call, every = _gdn().prefill_varlen, 64
    dd = to_dev(pk)
    args = (dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["cu"], dd["S0"])
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o32, S32, sn32 = call(*args, status=status, snap_every=every)
    o16, S16, sn16 = call(*args, status=status, snap_every=every, o_bf16=True)
    assert _gdn().query_status(status) == 0
    assert o16.dtype == torch.bfloat16
    assert torch.equal(o16, o32.to(torch.bfloat16))
    assert torch.equal(S16, S32) and torch.equal(sn16, sn32)


@pytest.mark.parametrize("gate", ["kda", "scalar"])
def test_varlen_many_sequences_keep_index_order(gate):
    """More sequences than a CTA has threads (520, of 0..40 tokens, one head):
    the longest-first ordering is skipped and every sequence still matches the
    oracle run on it alone."""
    rng = np.random.default_rng(950)
    lengths = [int(x) for x in rng.integers(0, 41, size=520)]
    if gate == "kda":
        seqs, pk = _kda_packed(lengths, 1, 128, seed=960, s0_std=0.05)
    else:
        seqs = [inputs.prefill_inputs(1, L, 1, seed=960 + i, s0_std=0.05) for i, L in enumerate(lengths)]
        cat = lambda key: torch.cat([d[key][0] for d in seqs], 0)
        pk = dict(q=cat("q"), k=cat("k"), v=cat("v"), g=cat("g"), beta=cat("beta"),
                  S0=torch.cat([d["S0"] for d in seqs], 0),
                  cu=torch.tensor([0] + list(np.cumsum(lengths)), dtype=torch.int32))
    dd = to_dev(pk)
    gdn = _gdn()
    call = gdn.kda_prefill_varlen if gate == "kda" else gdn.prefill_varlen
    ref = oracle.kda_prefill if gate == "kda" else oracle.prefill
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, S_T = call(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["cu"], dd["S0"], status=status)
    assert gdn.query_status(status) == 0
    o, S_T = o.cpu().numpy(), S_T.cpu().numpy()
    cu = pk["cu"].numpy()
    for n in range(0, 520, 7):
        d = seqs[n]
        if not lengths[n]:
            np.testing.assert_array_equal(S_T[n], d["S0"][0].numpy())
            continue
        ro, rS = ref(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
        assert_parity(o[cu[n]:cu[n + 1]], ro[0], f"o seq {n} (len {lengths[n]})")
        assert_parity(S_T[n], rS[0], f"S_T seq {n} (len {lengths[n]})")
