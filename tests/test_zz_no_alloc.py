"""gdn_prefill_static_ws (segmented prefill on the library's built-in device
scratch, no allocation) against gdn_prefill_ws with a caller workspace and
against the fp64 oracle, on two calls in a row; the state updated in place;
the size limit; and the single-pass shapes that need no scratch.  Collected
last on purpose: it must pass alone in a fresh process and after every other
test."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_linear_20_b200 import inputs

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
REL_FRO = 2e-3
MAXABS_FRAC = 1e-2


def _gdn():
    from gated_deltanet_linear_20_b200 import gdn
    return gdn


def assert_close(got, ref, what):
    got = got.double().cpu().numpy()
    ref = ref.double().cpu().numpy()
    assert np.isfinite(got).all(), what
    rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300)
    rms = np.sqrt(np.mean(ref * ref))
    mx = np.abs(got - ref).max() / max(rms, 1e-300)
    assert rel <= REL_FRO and mx <= MAXABS_FRAC, f"{what}: rel_fro={rel:.3e} maxabs/rms={mx:.3e}"


@pytest.mark.parametrize("B,T,H,chunk,s0", [
    (1, 512, 16, 64, 0.0),     # the single-sequence prefill workload (12 MiB of scratch)
    (1, 512, 16, 16, 0.0),
    (1, 577, 3, 64, 0.05),     # ragged last segment, carried state
])
def test_static_scratch_matches_caller_workspace_twice(B, T, H, chunk, s0):
    gdn = _gdn()
    need = gdn.workspace_bytes(B, T, H, chunk)
    assert 0 < need <= gdn.STATIC_WORKSPACE_BYTES
    d = inputs.prefill_inputs(B, T, H, seed=T + H, s0_std=s0, device=DEV)
    o_ref, S_ref = gdn.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], chunk=chunk)
    for call in range(2):
        status = torch.zeros(1, dtype=torch.int32, device=DEV)
        o, S_T = gdn.prefill_static(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"],
                                    chunk=chunk, status=status)
        assert gdn.query_status(status) == 0
        assert_close(o, o_ref, f"o, call {call}")
        assert_close(S_T, S_ref, f"S_T, call {call}")


@pytest.mark.parametrize("B,T,H,chunk,s0", [
    (1, 512, 16, 64, 0.0),
    (1, 577, 3, 16, 0.05),
])
def test_static_scratch_matches_the_oracle_twice(B, T, H, chunk, s0):
    gdn = _gdn()
    assert 0 < gdn.workspace_bytes(B, T, H, chunk) <= gdn.STATIC_WORKSPACE_BYTES
    d = inputs.prefill_inputs(B, T, H, seed=3 * T + H, s0_std=s0)
    ro, rS = oracle.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    dd = {k: (v.to(DEV) if v is not None else None) for k, v in d.items()}
    for call in range(2):
        status = torch.zeros(1, dtype=torch.int32, device=DEV)
        o, S_T = gdn.prefill_static(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["S0"],
                                    chunk=chunk, status=status)
        assert gdn.query_status(status) == 0
        assert_close(o, torch.from_numpy(ro), f"o vs oracle, call {call}")
        assert_close(S_T, torch.from_numpy(rS), f"S_T vs oracle, call {call}")


def test_static_scratch_state_in_place():
    """S_T is S0 on a segmented shape: segment 0 reads S0 in the first launch,
    and the second launch writes S_T over it."""
    gdn = _gdn()
    B, T, H = 1, 577, 3
    assert gdn.schedule(B, T, H, torch.cuda.get_device_properties(0).multi_processor_count)[0] > 1
    d = inputs.prefill_inputs(B, T, H, seed=11, s0_std=0.05)
    ro, rS = oracle.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    dd = {k: (v.to(DEV) if v is not None else None) for k, v in d.items()}
    S = dd["S0"].clone()
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, S_T = gdn.prefill_static(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], S, S_T=S,
                                status=status)
    assert gdn.query_status(status) == 0
    assert S_T.data_ptr() == S.data_ptr()
    assert_close(o, torch.from_numpy(ro), "o (state in place)")
    assert_close(S, torch.from_numpy(rS), "S_T written over S0")


def test_static_scratch_limit_is_reported():
    gdn = _gdn()
    B, T, H = 1, 4096, 16              # the long-prefill workload needs ~42 MiB
    assert gdn.workspace_bytes(B, T, H) > gdn.STATIC_WORKSPACE_BYTES
    d = inputs.prefill_inputs(B, T, H, seed=1, device=DEV)
    with pytest.raises(gdn.GDNError) as e:
        gdn.prefill_static(d["q"], d["k"], d["v"], d["g"], d["beta"])
    assert e.value.code == gdn.GDN_ERR_STATIC_WORKSPACE_LIMIT


def test_static_scratch_single_pass_shape_needs_none():
    gdn = _gdn()
    B, T, H = 4, 200, 32               # 128 chains: the single-pass schedule
    assert gdn.workspace_bytes(B, T, H) == 0
    d = inputs.prefill_inputs(B, T, H, seed=2, s0_std=0.02, device=DEV)
    a = gdn.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], segmented=False)
    b = gdn.prefill_static(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
