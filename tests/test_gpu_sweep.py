"""A seeded sweep of shapes and options through every entry point, each case
against the fp64 oracle (the contract and the 1e-4 design margin of the other
GPU tests).  The cases are drawn once from a fixed generator, so the sweep is
the same on every run; each is small enough for the oracle to finish in well
under a second.  What the sweep varies, per entry point:
  * gdn_prefill / gdn_prefill_ws: B, H, T (ragged, 1 .. 300), chunk 16 / 64,
    single pass / segmented, with or without S0, head dims {64, 128, 256}^2,
    gate strength (logsigmoid(N(mu, 1)), mu in {-3, 0, 2});
  * gdn_kda_prefill: B, H, T, with or without S0, the same gate strengths;
  * gdn_decode_tokens / gdn_kda_decode: B, H, T in 1 .. 6, head dims 64 / 128;
  * gdn_prefill_varlen: 1 .. 5 packed sequences of 0 .. 200 tokens, at 128 x 128
    and at the other tensor-core head dims;
  * the fused options (q/k L2 norm with a q scale, bf16 o) at the tensor-core
    head dims, prefill and decode.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_linear_20_b200 import inputs
from tests.test_gpu_parity import DEV, assert_parity, raw_qk, to_dev

pytestmark = pytest.mark.gpu

DIMS = (64, 128, 256)
GMEANS = (-3.0, 0.0, 2.0)


def _gdn():
    from gated_deltanet_linear_20_b200 import gdn
    return gdn


def _draw(n, seed, fn):
    rng = np.random.default_rng(seed)
    return [fn(rng, i) for i in range(n)]


PREFILL_CASES = _draw(48, 2024, lambda r, i: dict(
    B=int(r.integers(1, 3)), H=int(r.integers(1, 4)), T=int(r.integers(1, 301)),
    chunk=int(r.choice([16, 64])), segmented=bool(r.integers(0, 2)), s0=bool(r.integers(0, 2)),
    dk=int(r.choice(DIMS)), dv=int(r.choice(DIMS)), g_mean=float(r.choice(GMEANS)), seed=100 + i))


@pytest.mark.parametrize("case", PREFILL_CASES, ids=lambda c: "B{B}H{H}T{T}c{chunk}{seg}{s0}_{dk}x{dv}_g{g_mean:+.0f}".format(
    seg="s" if c["segmented"] else "p", s0="S0" if c["s0"] else "", **{k: v for k, v in c.items() if k not in ("segmented", "s0")}))
def test_prefill_sweep(case):
    c = case
    d = inputs.prefill_inputs(c["B"], c["T"], c["H"], c["dk"], c["dv"], seed=c["seed"],
                              g_mean=c["g_mean"], s0_std=0.05 if c["s0"] else None)
    dd = to_dev(d)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    gdn = _gdn()
    o, S_T = gdn.prefill(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["S0"], chunk=c["chunk"],
                         segmented=c["segmented"], status=status)
    assert gdn.query_status(status) == 0
    ro, rS = oracle.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    assert_parity(o.cpu().numpy(), ro, "o")
    assert_parity(S_T.cpu().numpy(), rS, "S_T")


KDA_CASES = _draw(24, 77, lambda r, i: dict(
    B=int(r.integers(1, 3)), H=int(r.integers(1, 4)), T=int(r.integers(1, 301)),
    s0=bool(r.integers(0, 2)), g_mean=float(r.choice(GMEANS)), seed=300 + i))


@pytest.mark.parametrize("case", KDA_CASES, ids=lambda c: "B{B}H{H}T{T}{s0}_g{g_mean:+.0f}".format(
    s0="S0" if c["s0"] else "", **{k: v for k, v in c.items() if k != "s0"}))
def test_kda_prefill_sweep(case):
    c = case
    d = inputs.kda_inputs(c["B"], c["T"], c["H"], seed=c["seed"], g_mean=c["g_mean"],
                          s0_std=0.05 if c["s0"] else None)
    dd = to_dev(d)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    gdn = _gdn()
    o, S_T = gdn.kda_prefill(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["S0"], status=status)
    assert gdn.query_status(status) == 0
    ro, rS = oracle.kda_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    assert_parity(o.cpu().numpy(), ro, "o")
    assert_parity(S_T.cpu().numpy(), rS, "S_T")


DECODE_CASES = _draw(24, 5, lambda r, i: dict(
    B=int(r.integers(1, 9)), H=int(r.integers(1, 5)), T=int(r.integers(1, 7)),
    D=int(r.choice([64, 128])), kda=bool(r.integers(0, 2)), g_mean=float(r.choice(GMEANS)),
    seed=500 + i))


@pytest.mark.parametrize("case", DECODE_CASES, ids=lambda c: "B{B}H{H}T{T}_D{D}_{gate}_g{g_mean:+.0f}".format(
    gate="kda" if c["kda"] else "scalar", **{k: v for k, v in c.items() if k != "kda"}))
def test_decode_sweep(case):
    """T tokens in one call (T = 1: the step kernel), the state in place."""
    c = case
    gen = inputs.kda_inputs if c["kda"] else inputs.prefill_inputs
    d = gen(c["B"], c["T"], c["H"], c["D"], c["D"], seed=c["seed"], g_mean=c["g_mean"], s0_std=0.05)
    dd = to_dev(d)
    gdn = _gdn()
    S = dd["S0"].clone()
    args = [dd[key] for key in ("q", "k", "v", "g", "beta")]
    o = gdn.kda_decode(*args, S) if c["kda"] else gdn.decode_tokens(*args, S)
    torch.cuda.synchronize()
    ref = oracle.kda_prefill if c["kda"] else oracle.prefill
    ro, rS = ref(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    assert_parity(o.cpu().numpy(), ro, "o")
    assert_parity(S.cpu().numpy(), rS, "S")


VARLEN_CASES = _draw(10, 9, lambda r, i: dict(
    lengths=[int(x) for x in r.integers(0, 201, size=int(r.integers(1, 6)))], H=int(r.integers(1, 4)),
    chunk=int(r.choice([16, 64])), s0=bool(r.integers(0, 2)), seed=700 + 10 * i))


@pytest.mark.parametrize("case", VARLEN_CASES, ids=lambda c: "L{}_H{}_c{}{}".format(
    "-".join(map(str, c["lengths"])), c["H"], c["chunk"], "S0" if c["s0"] else ""))
def test_varlen_sweep(case):
    c = case
    seqs = [inputs.prefill_inputs(1, L, c["H"], seed=c["seed"] + n, s0_std=0.05 if c["s0"] else None)
            for n, L in enumerate(c["lengths"])]
    cat = lambda key: torch.cat([s[key][0] for s in seqs], 0)
    S0 = torch.cat([s["S0"] for s in seqs], 0) if c["s0"] else None
    cu = torch.tensor([0] + list(np.cumsum(c["lengths"])), dtype=torch.int32)
    gdn = _gdn()
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, S_T = gdn.prefill_varlen(cat("q").to(DEV), cat("k").to(DEV), cat("v").to(DEV), cat("g").to(DEV),
                                cat("beta").to(DEV), cu.to(DEV), S0.to(DEV) if S0 is not None else None,
                                chunk=c["chunk"], status=status)
    assert gdn.query_status(status) == 0
    o = o.cpu().numpy()
    S_T = S_T.cpu().numpy()
    t0 = 0
    for n, (L, s) in enumerate(zip(c["lengths"], seqs)):
        ro, rS = oracle.prefill(s["q"], s["k"], s["v"], s["g"], s["beta"], s["S0"])
        if L:
            assert_parity(o[t0:t0 + L], ro[0], f"o of sequence {n}")
        assert_parity(S_T[n:n + 1], rS, f"S_T of sequence {n}")
        t0 += L


TC_DIMS = ((64, 64), (64, 128), (128, 64), (128, 128), (128, 256))

OPTION_CASES = _draw(16, 31, lambda r, i: dict(
    B=int(r.integers(1, 3)), H=int(r.integers(1, 4)), T=int(r.integers(1, 201)),
    chunk=int(r.choice([16, 64])), dims=TC_DIMS[int(r.integers(0, len(TC_DIMS)))],
    bf16=bool(r.integers(0, 2)), seed=900 + i))


@pytest.mark.parametrize("case", OPTION_CASES, ids=lambda c: "B{B}H{H}T{T}c{chunk}_{d[0]}x{d[1]}{o}".format(
    d=c["dims"], o="_bf16" if c["bf16"] else "", **{k: v for k, v in c.items() if k not in ("dims", "bf16")}))
def test_fused_options_sweep(case):
    """The fused q/k norm and q scale (and bf16 o) in the tensor-core prefill at
    a drawn head-dim pair, against the oracle on fp64-normalised inputs; bf16 o
    within one bf16 ulp of the oracle plus the fp32 path's tolerance."""
    c = case
    dk, dv = c["dims"]
    d = inputs.prefill_inputs(c["B"], c["T"], c["H"], dk, dv, seed=c["seed"], s0_std=0.05)
    r = raw_qk(d, c["seed"] + 1)
    qs = dk ** -0.5
    dd = to_dev(d)
    gdn = _gdn()
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, S_T = gdn.prefill(r["q"].to(DEV), r["k"].to(DEV), dd["v"], dd["g"], dd["beta"], dd["S0"],
                         chunk=c["chunk"], qk_l2norm=True, q_scale=qs, o_bf16=c["bf16"], status=status)
    assert gdn.query_status(status) == 0
    ro, rS = oracle.prefill((r["q_n"] * qs).float(), r["k_n"].float(), d["v"], d["g"], d["beta"], d["S0"])
    if c["bf16"]:
        got = o.float().cpu().numpy().astype(np.float64)
        ref = np.asarray(ro, dtype=np.float64)
        rms = float(np.sqrt(np.mean(ref ** 2)))
        assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -7 + 1e-2 * rms)
    else:
        assert_parity(o.cpu().numpy(), ro, "o")
    assert_parity(S_T.cpu().numpy(), rS, "S_T")


VARLEN_DIM_CASES = _draw(10, 13, lambda r, i: dict(
    lengths=[int(x) for x in r.integers(0, 161, size=int(r.integers(1, 5)))], H=int(r.integers(1, 3)),
    chunk=int(r.choice([16, 64])), dims=TC_DIMS[int(r.integers(0, len(TC_DIMS)))], seed=950 + 10 * i))


@pytest.mark.parametrize("case", VARLEN_DIM_CASES, ids=lambda c: "L{}_H{}_c{}_{}x{}".format(
    "-".join(map(str, c["lengths"])), c["H"], c["chunk"], *c["dims"]))
def test_varlen_head_dims_sweep(case):
    """Packed sequences at a drawn tensor-core head-dim pair, with carried
    states, each sequence against the oracle run on it alone."""
    c = case
    dk, dv = c["dims"]
    seqs = [inputs.prefill_inputs(1, L, c["H"], dk, dv, seed=c["seed"] + n, s0_std=0.05)
            for n, L in enumerate(c["lengths"])]
    cat = lambda key: torch.cat([s[key][0] for s in seqs], 0)
    S0 = torch.cat([s["S0"] for s in seqs], 0)
    cu = torch.tensor([0] + list(np.cumsum(c["lengths"])), dtype=torch.int32)
    gdn = _gdn()
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, S_T = gdn.prefill_varlen(cat("q").to(DEV), cat("k").to(DEV), cat("v").to(DEV), cat("g").to(DEV),
                                cat("beta").to(DEV), cu.to(DEV), S0.to(DEV), chunk=c["chunk"], status=status)
    assert gdn.query_status(status) == 0
    o = o.cpu().numpy()
    S_T = S_T.cpu().numpy()
    t0 = 0
    for n, (L, s) in enumerate(zip(c["lengths"], seqs)):
        ro, rS = oracle.prefill(s["q"], s["k"], s["v"], s["g"], s["beta"], s["S0"])
        if L:
            assert_parity(o[t0:t0 + L], ro[0], f"o of sequence {n}")
        assert_parity(S_T[n:n + 1], rS, f"S_T of sequence {n}")
        t0 += L
