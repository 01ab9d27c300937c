"""The seeded input generators (CPU): shapes, dtypes, determinism and the
recipe's distributions and draw order.  These are the only code that the
oracle and the CUDA path share, so their recipe is pinned here."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from gated_deltanet_linear_20_b200 import inputs


def test_prefill_inputs_shapes_dtypes_and_determinism():
    a = inputs.prefill_inputs(2, 7, 3, 64, 256, seed=5, s0_std=0.1)
    b = inputs.prefill_inputs(2, 7, 3, 64, 256, seed=5, s0_std=0.1)
    c = inputs.prefill_inputs(2, 7, 3, 64, 256, seed=6, s0_std=0.1)
    assert a["q"].shape == (2, 7, 3, 64) and a["q"].dtype == torch.bfloat16
    assert a["k"].shape == (2, 7, 3, 64) and a["v"].shape == (2, 7, 3, 256)
    assert a["v"].dtype == torch.bfloat16
    assert a["g"].shape == (2, 7, 3) and a["g"].dtype == torch.float32
    assert a["beta"].shape == (2, 7, 3) and a["S0"].shape == (2, 3, 256, 64)
    for key in a:
        assert torch.equal(a[key], b[key]), key
    assert not torch.equal(a["q"], c["q"])


def test_prefill_inputs_distributions():
    d = inputs.prefill_inputs(1, 256, 4, seed=1, s0_std=0.02)
    for key in ("q", "k"):
        n = d[key].double().norm(dim=-1)
        assert torch.allclose(n, torch.ones_like(n), atol=1e-2), key  # unit norm up to bf16
    g = d["g"]
    assert (g < 0).all() and g.mean().item() == pytest.approx(-0.81, abs=0.1)  # logsigmoid(N(0,1))
    assert ((d["beta"] > 0) & (d["beta"] < 1)).all()
    assert d["S0"].std().item() == pytest.approx(0.02, rel=0.05)
    assert inputs.prefill_inputs(1, 4, 1, seed=0)["S0"] is None
    slow = inputs.prefill_inputs(1, 256, 4, seed=1, g_mean=2.0)["g"]
    assert slow.mean().item() > -0.3  # long memory: alpha close to 1


def test_kda_inputs_share_the_recipe_and_draw_a_gate_per_channel():
    """Draw order q, k, v, g_raw, beta_raw, S0: q, k, v equal the scalar-gate
    draws for the same seed; g is [B,T,H,Dk] and differs across channels."""
    p = inputs.prefill_inputs(2, 9, 3, 128, 64, seed=11)
    k = inputs.kda_inputs(2, 9, 3, 128, 64, seed=11, s0_std=0.05)
    for key in ("q", "k", "v"):
        assert torch.equal(p[key], k[key]), key
    assert k["g"].shape == (2, 9, 3, 128) and k["g"].dtype == torch.float32
    assert (k["g"] < 0).all()
    assert k["g"].std(dim=-1).min().item() > 0.1  # not one value broadcast over channels
    assert k["beta"].shape == (2, 9, 3) and k["S0"].shape == (2, 3, 64, 128)
    again = inputs.kda_inputs(2, 9, 3, 128, 64, seed=11, s0_std=0.05)
    for key in k:
        assert torch.equal(k[key], again[key]), key


def test_decode_inputs_are_the_prefill_draws_step_major():
    d = inputs.decode_inputs(3, 2, 5, seed=4, s0_std=0.02)
    p = inputs.prefill_inputs(3, 5, 2, seed=4, s0_std=0.02)
    assert d["q"].shape == (5, 3, 2, 128)
    assert torch.equal(d["q"], p["q"].transpose(0, 1))
    assert torch.equal(d["g"], p["g"].transpose(0, 1))
    assert torch.equal(d["S"], p["S0"])


def test_workloads_have_the_stated_shapes():
    w = inputs.WORKLOADS
    assert (w["prefill_b1_h16_t512"].B, w["prefill_b1_h16_t512"].H, w["prefill_b1_h16_t512"].T) == (1, 16, 512)
    assert w["decode_b64_h16"].is_decode and w["decode_b64_h16"].decode_steps == 256
    assert w["prefill_b4_h32_t32768"].g_mean == 2.0
    assert w["prefill_b1_h16_t4096_s0"].s0_std == 0.02
    for wl in w.values():
        assert wl.Dk == 128 and wl.Dv == 128
        assert wl.describe()
