"""Pins for the per-channel-gate (KDA) oracle, CPU only.

The ROCmFPX gated-delta-net prefill note (bittide.aicompass.dev article
d2880479, opening post) names KDA as a case its fused kernel left to the old
path; it prints no formula.  The oracle takes the plainest reading: the
scalar gate alpha_t of the gated delta rule becomes a decay per key channel,
applied where the scalar one is,

    S_t = S_{t-1} diag(alpha_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
    o_t = S_t q_t,  alpha_t = exp(g_t) in R^{Dk},

with S in R^{Dv x Dk}.  The pins below follow from that definition:

* reduction: a gate equal on every channel is the scalar gated delta rule
  (whose oracle is pinned on its own in test_oracle_pins.py);
* closed form: beta = 0 decays column j of S0 by exp(sum_t g_tj) -- columns,
  not rows, since Dk != Dv and the channel decays differ;
* the delta-rule write: beta = 1 with an exactly unit key stores v_t
  (S_t k_t = v_t, read through o_t with q_t = k_t), which fails if the decay
  sits after the projection instead of before it;
* brute force: dense ordered matrix products for T <= 7;
* the chunked form with per-channel cumulative decays Lambda_i = exp(gamma_i):
  K+ = K o Lambda, K- = K / Lambda, Q+ = Q o Lambda,
  A = tril(diag(beta) K+ K-^T, -1), U = (I + A)^-1 diag(beta)(V - K+ S_c^T),
  O = Q+ S_c^T + tril(Q+ K-^T) U,
  S_next = S_c diag(Lambda_C) + U^T (K o Lambda_C / Lambda),
  derived here independently and written in numpy fp64;
* structure: split-T carry, padding tokens (k = 0, beta = 0, g = 0) as the
  identity, and equivariance under a permutation of the key channels.

The last test plants mistakes in a copy of the oracle and checks that each
fails some pin.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import tempfile

import numpy as np
import pytest

import oracle

RTOL = 1e-11


def _case(B=1, T=12, H=2, Dk=8, Dv=5, seed=0, s0=True, unit_k=True):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, H, Dk)).astype(np.float32)
    k = rng.standard_normal((B, T, H, Dk)).astype(np.float32)
    if unit_k:
        k = (k / np.linalg.norm(k, axis=-1, keepdims=True)).astype(np.float32)
    v = rng.standard_normal((B, T, H, Dv)).astype(np.float32)
    g = (-rng.uniform(0.01, 1.0, (B, T, H, Dk))).astype(np.float32)
    beta = rng.uniform(0.0, 1.0, (B, T, H)).astype(np.float32)
    S0 = (0.3 * rng.standard_normal((B, H, Dv, Dk))).astype(np.float32) if s0 else None
    return q, k, v, g, beta, S0


def _rel(a, b):
    return float(np.linalg.norm(np.asarray(a) - np.asarray(b)) / max(np.linalg.norm(b), 1e-300))


# ----------------------------------------------------------------------------------------
# independent restatements (numpy fp64, test code only)

def _brute_force_chain(q, k, v, g, beta, S0):
    """S_t = S0 M_1..M_t + sum_r beta_r v_r k_r^T M_{r+1}..M_t with
    M_s = diag(exp(g_s)) (I - beta_s k_s k_s^T).  q,k,g [T,Dk]; v [T,Dv]; beta [T]."""
    T, Dk = k.shape
    Dv = v.shape[1]
    q, k, v, g, beta = (x.astype(np.float64) for x in (q, k, v, g, beta))
    M = [np.diag(np.exp(g[s])) @ (np.eye(Dk) - beta[s] * np.outer(k[s], k[s])) for s in range(T)]
    o = np.zeros((T, Dv))
    S_t = None
    for t in range(T):
        P = np.eye(Dk)
        for s in range(t + 1):
            P = P @ M[s]
        S_t = S0.astype(np.float64) @ P
        for r in range(t + 1):
            R = np.eye(Dk)
            for s in range(r + 1, t + 1):
                R = R @ M[s]
            S_t = S_t + beta[r] * np.outer(v[r], k[r]) @ R
        o[t] = S_t @ q[t]
    return o, S_t


def _chunked_chain(q, k, v, g, beta, S0, C):
    """The chunked form with per-channel decays (see the module docstring)."""
    q, k, v, g, beta = (x.astype(np.float64) for x in (q, k, v, g, beta))
    T, Dk = k.shape
    S = S0.astype(np.float64).copy()
    o = np.zeros((T, v.shape[1]))
    for c0 in range(0, T, C):
        sl = slice(c0, min(c0 + C, T))
        K, Q, V, bb = k[sl], q[sl], v[sl], beta[sl]
        n = K.shape[0]
        lam = np.exp(np.cumsum(g[sl], axis=0))                 # [n, Dk], Lambda_i
        Kp, Km, Qp = K * lam, K / lam, Q * lam
        A = np.tril(bb[:, None] * (Kp @ Km.T), -1)
        U = np.linalg.solve(np.eye(n) + A, bb[:, None] * (V - Kp @ S.T))
        o[sl] = Qp @ S.T + np.tril(Qp @ Km.T) @ U
        S = S * lam[-1][None, :] + U.T @ (K * (lam[-1][None, :] / lam))
    return o, S


# ----------------------------------------------------------------------------------------
# the pins, each against a kda(q,k,v,g,beta,S0) -> (o, S_T) callable

def pin_scalar_gate_reduction(kda):
    q, k, v, g, beta, S0 = _case(seed=1)
    gs = g[..., 0]
    o, S_T = kda(q, k, v, np.ascontiguousarray(np.repeat(gs[..., None], g.shape[-1], -1)), beta, S0)
    ro, rS = oracle.prefill(q, k, v, gs, beta, S0)
    return _rel(o, ro) < RTOL and _rel(S_T, rS) < RTOL


def pin_beta0_column_decay(kda):
    q, k, v, g, beta, S0 = _case(seed=2)
    beta[:] = 0
    o, S_T = kda(q, k, v, g, beta, S0)
    G = np.cumsum(g.astype(np.float64), axis=1)                      # [B,T,H,Dk]
    S0d = S0.astype(np.float64)
    ref_S = S0d * np.exp(G[:, -1])[:, :, None, :]
    ref_o = np.einsum("bhij,bthj,bthj->bthi", S0d, np.exp(G), q.astype(np.float64))
    return _rel(S_T, ref_S) < RTOL and _rel(o, ref_o) < RTOL


def _exact_unit_keys(rng, shape_btH, Dk):
    """Keys with four entries of +-1/2 and zeros elsewhere: unit norm exactly."""
    B, T, H = shape_btH
    k = np.zeros((B, T, H, Dk), np.float32)
    for idx in np.ndindex(B, T, H):
        pos = rng.choice(Dk, 4, replace=False)
        k[idx][pos] = rng.choice([-0.5, 0.5], 4)
    return k


def pin_beta1_writes_value(kda):
    rng = np.random.default_rng(3)
    q, k, v, g, beta, S0 = _case(seed=3, T=10)
    k = _exact_unit_keys(rng, beta.shape, k.shape[-1])
    beta[:] = 1
    o, _ = kda(k.copy(), k, v, g, beta, S0)                          # q_t = k_t -> o_t = S_t k_t
    return np.allclose(o, v.astype(np.float64), rtol=0, atol=1e-12)


def pin_brute_force(kda):
    q, k, v, g, beta, S0 = _case(B=1, T=7, H=2, Dk=6, Dv=4, seed=4, unit_k=False)
    o, S_T = kda(q, k, v, g, beta, S0)
    for h in range(2):
        ro, rS = _brute_force_chain(q[0, :, h], k[0, :, h], v[0, :, h], g[0, :, h], beta[0, :, h],
                                    S0[0, h])
        if _rel(o[0, :, h], ro) > 1e-10 or _rel(S_T[0, h], rS) > 1e-10:
            return False
    return True


def pin_chunked_form(kda):
    q, k, v, g, beta, S0 = _case(B=1, T=37, H=2, Dk=8, Dv=5, seed=5)
    o, S_T = kda(q, k, v, g, beta, S0)
    for C in (1, 4, 16):
        for h in range(2):
            ro, rS = _chunked_chain(q[0, :, h], k[0, :, h], v[0, :, h], g[0, :, h], beta[0, :, h],
                                    S0[0, h], C)
            if _rel(o[0, :, h], ro) > 1e-9 or _rel(S_T[0, h], rS) > 1e-9:
                return False
    return True


def pin_split_carry(kda):
    q, k, v, g, beta, S0 = _case(T=23, seed=6)
    o, S_T = kda(q, k, v, g, beta, S0)
    t1 = 9
    o1, S1 = kda(q[:, :t1], k[:, :t1], v[:, :t1], g[:, :t1], beta[:, :t1], S0)
    o2, S2 = kda(q[:, t1:], k[:, t1:], v[:, t1:], g[:, t1:], beta[:, t1:], S1.astype(np.float32))
    return _rel(np.concatenate([o1, o2], 1), o) < 1e-6 and _rel(S2, S_T) < 1e-6 and \
        _rel(o1, o[:, :t1]) < RTOL


def pin_padding_identity(kda):
    q, k, v, g, beta, S0 = _case(T=11, seed=10)
    o, S_T = kda(q, k, v, g, beta, S0)
    pad = 5
    rng = np.random.default_rng(10)
    qp = np.concatenate([q, rng.standard_normal(q[:, :pad].shape).astype(np.float32)], 1)
    kp = np.concatenate([k, np.zeros_like(k[:, :pad])], 1)
    vp = np.concatenate([v, rng.standard_normal(v[:, :pad].shape).astype(np.float32)], 1)
    gp = np.concatenate([g, np.zeros_like(g[:, :pad])], 1)
    bp = np.concatenate([beta, np.zeros_like(beta[:, :pad])], 1)
    o2, S2 = kda(qp, kp, vp, gp, bp, S0)
    return np.array_equal(S2, S_T) and np.array_equal(o2[:, :11], o)


def pin_key_channel_permutation(kda):
    """Relabelling the key channels (q, k, g and the columns of S0 together)
    leaves o unchanged and permutes the columns of S_T."""
    q, k, v, g, beta, S0 = _case(seed=9)
    perm = np.random.default_rng(9).permutation(k.shape[-1])
    o, S_T = kda(q, k, v, g, beta, S0)
    c = lambda x: np.ascontiguousarray(x[..., perm])
    op, Sp = kda(c(q), c(k), v, c(g), beta, c(S0))
    return _rel(op, o) < 1e-13 and _rel(Sp, S_T[..., perm]) < 1e-13


PINS = [pin_scalar_gate_reduction, pin_beta0_column_decay, pin_beta1_writes_value,
        pin_brute_force, pin_chunked_form, pin_split_carry, pin_padding_identity,
        pin_key_channel_permutation]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_kda_oracle_pin(pin):
    assert pin(oracle.kda_prefill)


def test_kda_full_head_dim_brute_force():
    """Head dim 128 against the dense-product brute force, T = 4, Dk != Dv."""
    q, k, v, g, beta, S0 = _case(B=1, T=4, H=1, Dk=128, Dv=96, seed=15)
    o, S_T = oracle.kda_prefill(q, k, v, g, beta, S0)
    ro, rS = _brute_force_chain(q[0, :, 0], k[0, :, 0], v[0, :, 0], g[0, :, 0], beta[0, :, 0],
                                S0[0, 0])
    assert _rel(o[0, :, 0], ro) < 1e-11 and _rel(S_T[0, 0], rS) < 1e-11


def test_kda_zero_initial_state_is_none():
    q, k, v, g, beta, S0 = _case(seed=16)
    o1, S1 = oracle.kda_prefill(q, k, v, g, beta, None)
    o2, S2 = oracle.kda_prefill(q, k, v, g, beta, np.zeros_like(S0))
    assert np.array_equal(o1, o2) and np.array_equal(S1, S2)


# ----------------------------------------------------------------------------------------
# mutation check: each plausible mistake planted in a copy of the oracle fails some pin

MUTANTS = {
    "decay_on_rows": [("Si[j] = a[j] * Si[j] - bt", "Si[j] = a[i % Dk] * Si[j] - bt")],
    "projection_ungated": [("acc += Si[j] * a[j] * (double)kt[j];", "acc += Si[j] * (double)kt[j];")],
    "decay_after_projection": [
        ("acc += Si[j] * a[j] * (double)kt[j];", "acc += Si[j] * (double)kt[j];"),
        ("Si[j] = a[j] * Si[j] - bt * u[i] * kj + bt * vi * kj;",
         "Si[j] = a[j] * (Si[j] - bt * u[i] * kj) + bt * vi * kj;")],
    "negated_gate": [("a[j] = exp((double)gt[j]);", "a[j] = exp(-(double)gt[j]);")],
    "gate_of_channel0": [("a[j] = exp((double)gt[j]);", "a[j] = exp((double)gt[0]);")],
    "gate_of_token0": [("g + idx4(b, t, h, 0, T, H, Dk)", "g + idx4(b, 0, h, 0, T, H, Dk)")],
    "correction_sign": [("Si[j] = a[j] * Si[j] - bt * u[i] * kj",
                         "Si[j] = a[j] * Si[j] + bt * u[i] * kj")],
    "beta_dropped_on_write": [("- bt * u[i] * kj + bt * vi * kj;", "- bt * u[i] * kj + vi * kj;")],
    "gate_dropped_on_state": [("Si[j] = a[j] * Si[j] - bt", "Si[j] = Si[j] - bt")],
    "beta_of_head0": [("(double)beta[gi], o + idx4", "(double)beta[gi - h], o + idx4")],
}


def _load_kda_from(path):
    lib = ctypes.CDLL(path)
    fp = ctypes.POINTER(ctypes.c_float)
    dp = ctypes.POINTER(ctypes.c_double)
    lib.oracle_kda_prefill_f64.argtypes = [fp] * 6 + [dp, dp] + [ctypes.c_int] * 5
    lib.oracle_kda_prefill_f64.restype = ctypes.c_int

    def kda(q, k, v, g, beta, S0=None):
        arrs = [np.ascontiguousarray(np.asarray(x, np.float32)) if x is not None else None
                for x in (q, k, v, g, beta, S0)]
        B, T, H, Dk = arrs[0].shape
        Dv = arrs[2].shape[-1]
        o = np.empty((B, T, H, Dv))
        S_T = np.empty((B, H, Dv, Dk))
        ptrs = [a.ctypes.data_as(fp) if a is not None else None for a in arrs]
        rc = lib.oracle_kda_prefill_f64(*ptrs, o.ctypes.data_as(dp), S_T.ctypes.data_as(dp),
                                        B, T, H, Dk, Dv)
        assert rc == 0
        return o, S_T
    return kda


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_every_planted_kda_mistake_fails_a_pin(name):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "gdn_oracle.c")).read()
    for old, new in MUTANTS[name]:
        assert src.count(old) == 1, f"mutation anchor for {name} not unique: {old}"
        src = src.replace(old, new)
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "m.c")
        so = os.path.join(d, "m.so")
        open(c, "w").write(src)
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-std=c99", "-o", so, c, "-lm"])
        kda = _load_kda_from(so)
        results = {p.__name__: bool(p(kda)) for p in PINS}
    assert not all(results.values()), f"mutant {name} passed every pin: {results}"


def test_empty_shapes():
    """T = 0 leaves the state (S_T = S0, or zeros); B = 0 or H = 0 returns empty
    arrays; both oracles agree on it."""
    q, k, v, g, beta, S0 = _case(B=2, T=0, H=3, Dk=8, Dv=5, seed=17)
    for f, gg in ((oracle.kda_prefill, g), (oracle.prefill, g[..., 0])):
        o, S_T = f(q, k, v, gg, beta, S0)
        assert o.shape == (2, 0, 3, 5) and np.array_equal(S_T, S0.astype(np.float64))
        o, S_T = f(q, k, v, gg, beta, None)
        assert not S_T.any()
    q, k, v, g, beta, S0 = _case(B=0, T=4, H=3, Dk=8, Dv=5, seed=18)
    o, S_T = oracle.kda_prefill(q, k, v, g, beta, S0)
    assert o.shape == (0, 4, 3, 5) and S_T.shape == (0, 3, 5, 8)
