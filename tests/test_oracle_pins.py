"""Pins for the fp64 oracle (CPU only).

The pages print no worked example for the gated delta rule, so the oracle is
pinned by what the mathematics of the recurrence fixes:

    S_t = alpha_t S_{t-1}(I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
    o_t = S_t q_t,  alpha_t = exp(g_t)

(the gated delta rule of the hybrid Qwen 3.5 linear-attention layers; setting
from the ROCmFPX gated-delta-net prefill note, bittide.aicompass.dev article
d2880479, opening post: scalar gate, head dim 128, state in F32).

* closed forms: beta = 0 with g = 0 leaves S0 untouched; beta = 0 gives a
  pure exponential decay of S0;
* the delta-rule write: beta = 1 with an exactly unit-norm k_t stores v_t,
  S_t k_t = v_t (checked through o_t with q_t = k_t);
* brute force: dense ordered matrix products for T <= 8, and exact rational
  arithmetic (fractions.Fraction) on a 3x2 state;
* structure: split-T carry, superposition in (V, S0), Dv-row permutation
  equivariance, padding tokens as the identity, chain independence, decode
  step == prefill with T = 1;
* the chunked WY/UT form of the same recurrence, written here independently in
  numpy fp64, agrees with the oracle for chunk sizes 1, 4, 16 and 64 with
  ragged tails.

Dk != Dv throughout so that a transposed state cannot pass.  The last test
compiles mutants of the oracle (a dropped term, a wrong sign, a transposed
operand, a wrong index ...) and checks that every one fails some pin.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import tempfile
from fractions import Fraction

import numpy as np
import pytest

import oracle

RTOL = 1e-11


def _case(B=1, T=12, H=2, Dk=8, Dv=5, seed=0, s0=True, unit_k=True, g_scale=1.0):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, H, Dk)).astype(np.float32)
    k = rng.standard_normal((B, T, H, Dk)).astype(np.float32)
    if unit_k:
        k = (k / np.linalg.norm(k, axis=-1, keepdims=True)).astype(np.float32)
    v = rng.standard_normal((B, T, H, Dv)).astype(np.float32)
    g = (-g_scale * rng.uniform(0.01, 1.0, (B, T, H))).astype(np.float32)
    beta = rng.uniform(0.0, 1.0, (B, T, H)).astype(np.float32)
    S0 = (0.3 * rng.standard_normal((B, H, Dv, Dk))).astype(np.float32) if s0 else None
    return q, k, v, g, beta, S0


def _rel(a, b):
    return float(np.linalg.norm(np.asarray(a) - np.asarray(b)) / max(np.linalg.norm(b), 1e-300))


# ----------------------------------------------------------------------------------------
# independent restatements used as pins (numpy fp64, test code only)

def _brute_force_chain(q, k, v, g, beta, S0):
    """Dense ordered products: S_t = S0 M_1..M_t + sum_r beta_r v_r k_r^T M_{r+1}..M_t,
    M_s = alpha_s (I - beta_s k_s k_s^T).  q,k [T,Dk]; v [T,Dv]; g, beta [T]."""
    T, Dk = k.shape
    Dv = v.shape[1]
    q, k, v, g, beta = (x.astype(np.float64) for x in (q, k, v, g, beta))
    M = [np.exp(g[s]) * (np.eye(Dk) - beta[s] * np.outer(k[s], k[s])) for s in range(T)]
    o = np.zeros((T, Dv))
    S_t = None
    for t in range(T):
        P = np.eye(Dk)
        for s in range(t + 1):
            P = P @ M[s]
        S_t = (S0.astype(np.float64) @ P) if S0 is not None else np.zeros((Dv, Dk))
        for r in range(t + 1):
            R = np.eye(Dk)
            for s in range(r + 1, t + 1):
                R = R @ M[s]
            S_t = S_t + beta[r] * np.outer(v[r], k[r]) @ R
        o[t] = S_t @ q[t]
    return o, S_t


def _chunked_chain(q, k, v, g, beta, S0, C):
    """The chunked (WY/UT) form: within a chunk with gamma = cumsum(g),
    A = tril(diag(beta) K K^T * exp(gamma_i - gamma_j), -1), T = (I + A)^-1,
    Delta = T (diag(beta) V - diag(beta e^gamma) K S_c^T),
    O = diag(e^gamma) Q S_c^T + tril(Q K^T * exp(gamma_i - gamma_j)) Delta,
    S_next = e^{gamma_C} S_c + Delta^T diag(e^{gamma_C - gamma}) K."""
    q, k, v, g, beta = (x.astype(np.float64) for x in (q, k, v, g, beta))
    T, Dk = k.shape
    Dv = v.shape[1]
    S = np.zeros((Dv, Dk)) if S0 is None else S0.astype(np.float64).copy()
    o = np.zeros((T, Dv))
    for c0 in range(0, T, C):
        sl = slice(c0, min(c0 + C, T))
        K, Q, V, gg, bb = k[sl], q[sl], v[sl], g[sl], beta[sl]
        n = len(gg)
        gam = np.cumsum(gg)
        expo = np.tril(gam[:, None] - gam[None, :])
        Dec = np.tril(np.exp(expo))
        A = np.tril(bb[:, None] * (K @ K.T) * Dec, -1)
        Tm = np.linalg.inv(np.eye(n) + A)
        X = bb[:, None] * V - (bb * np.exp(gam))[:, None] * (K @ S.T)
        Delta = Tm @ X
        o[sl] = np.exp(gam)[:, None] * (Q @ S.T) + (np.tril(Q @ K.T) * Dec) @ Delta
        d = np.exp(gam[-1] - gam)
        S = np.exp(gam[-1]) * S + (Delta * d[:, None]).T @ K
    return o, S


def _rational_chain(q, k, v, alpha, beta, S0):
    """Exact arithmetic over Fractions; every input a Fraction."""
    T, Dk, Dv = len(k), len(k[0]), len(v[0])
    S = [row[:] for row in S0]
    outs = []
    for t in range(T):
        u = [sum(S[i][j] * k[t][j] for j in range(Dk)) for i in range(Dv)]
        S = [[alpha[t] * S[i][j] - alpha[t] * beta[t] * u[i] * k[t][j] + beta[t] * v[t][i] * k[t][j]
              for j in range(Dk)] for i in range(Dv)]
        outs.append([sum(S[i][j] * q[t][j] for j in range(Dk)) for i in range(Dv)])
    return outs, S


# ----------------------------------------------------------------------------------------
# the pin checks, written against a prefill(q,k,v,g,beta,S0) -> (o, S_T) callable so the
# mutation test can run them on broken oracles too.  Each returns True when the pin holds.

def pin_beta0_g0_constant(prefill):
    q, k, v, g, beta, S0 = _case(seed=1)
    g[:] = 0
    beta[:] = 0
    o, S_T = prefill(q, k, v, g, beta, S0)
    ok_S = np.allclose(S_T, S0.astype(np.float64), rtol=0, atol=1e-12)
    ref_o = np.einsum("bhij,bthj->bthi", S0.astype(np.float64), q.astype(np.float64))
    return ok_S and _rel(o, ref_o) < RTOL


def pin_beta0_decay_closed_form(prefill):
    q, k, v, g, beta, S0 = _case(seed=2)
    beta[:] = 0
    o, S_T = prefill(q, k, v, g, beta, S0)
    G = np.cumsum(g.astype(np.float64), axis=1)                      # [B,T,H]
    ref_S = np.exp(G[:, -1])[:, :, None, None] * S0
    ref_o = np.exp(G)[..., None] * np.einsum("bhij,bthj->bthi", S0.astype(np.float64),
                                              q.astype(np.float64))
    return _rel(S_T, ref_S) < RTOL and _rel(o, ref_o) < RTOL


def _exact_unit_keys(rng, shape_btH, Dk):
    """Keys with four entries of +-1/2 and zeros elsewhere: unit norm exactly."""
    B, T, H = shape_btH
    k = np.zeros((B, T, H, Dk), np.float32)
    for idx in np.ndindex(B, T, H):
        pos = rng.choice(Dk, 4, replace=False)
        k[idx][pos] = rng.choice([-0.5, 0.5], 4)
    return k


def pin_beta1_writes_value(prefill):
    rng = np.random.default_rng(3)
    q, k, v, g, beta, S0 = _case(seed=3, T=10)
    k = _exact_unit_keys(rng, g.shape, k.shape[-1])
    beta[:] = 1
    o, _ = prefill(k.copy(), k, v, g, beta, S0)                       # q_t = k_t -> o_t = S_t k_t
    return np.allclose(o, v.astype(np.float64), rtol=0, atol=1e-12)


def pin_brute_force(prefill):
    q, k, v, g, beta, S0 = _case(B=1, T=7, H=2, Dk=6, Dv=4, seed=4, unit_k=False)
    o, S_T = prefill(q, k, v, g, beta, S0)
    for h in range(2):
        ro, rS = _brute_force_chain(q[0, :, h], k[0, :, h], v[0, :, h], g[0, :, h], beta[0, :, h],
                                    S0[0, h])
        if _rel(o[0, :, h], ro) > 1e-10 or _rel(S_T[0, h], rS) > 1e-10:
            return False
    return True


def pin_exact_rational(prefill):
    # Dv=3, Dk=2, T=4.  The inputs are float32 numbers taken exactly as Fractions, so the
    # reference is the exact result.  alpha = 1 (g = 0) is exact; the case with alpha = 1/2
    # on alternate steps passes g = log(1/2) rounded to fp32 and is checked to 1e-6.
    F = lambda x: Fraction(float(np.float32(x)))
    kk = [[F(1), F(0)], [F(0.6), F(0.8)], [F(0), F(-1)], [F(-0.8), F(0.6)]]
    vv = [[F(1), F(-2), F(3)], [F(0.5), F(1), F(0)], [F(-1), F(0.25), F(2)], [F(0), F(3), F(-1)]]
    qq = [[F(2), F(1)], [F(-1), F(0.5)], [F(0.25), F(1)], [F(1), F(-1)]]
    bb = [F(0.5), F(0.25), F(0.75), F(1)]
    S0 = [[F(0.125), F(-0.25)], [F(0), F(0.5)], [F(0.375), F(0.125)]]
    ok = True
    for alphas, tol in (([Fraction(1)] * 4, 1e-14),
                        ([Fraction(1), Fraction(1, 2), Fraction(1), Fraction(1, 2)], 1e-6)):
        ro, rS = _rational_chain(qq, kk, vv, alphas, bb, S0)
        f = lambda rows: np.array([[float(x) for x in r] for r in rows], dtype=np.float64)
        q = f(qq).astype(np.float32)[None, :, None, :]
        k = f(kk).astype(np.float32)[None, :, None, :]
        v = f(vv).astype(np.float32)[None, :, None, :]
        g = np.log(np.array([float(a) for a in alphas])).astype(np.float32)[None, :, None]
        beta = np.array([float(b) for b in bb], np.float32)[None, :, None]
        s0 = f(S0).astype(np.float32)[None, None]
        o, S_T = prefill(q, k, v, g, beta, s0)
        ok &= _rel(o[0, :, 0], f(ro)) < tol and _rel(S_T[0, 0], f(rS)) < tol
    return ok


def pin_chunked_form(prefill):
    q, k, v, g, beta, S0 = _case(B=1, T=100, H=2, Dk=8, Dv=5, seed=5)
    o, S_T = prefill(q, k, v, g, beta, S0)
    for C in (1, 4, 16, 64):
        for h in range(2):
            ro, rS = _chunked_chain(q[0, :, h], k[0, :, h], v[0, :, h], g[0, :, h], beta[0, :, h],
                                    S0[0, h], C)
            if _rel(o[0, :, h], ro) > 1e-10 or _rel(S_T[0, h], rS) > 1e-10:
                return False
    return True


def pin_split_carry(prefill):
    q, k, v, g, beta, S0 = _case(T=23, seed=6)
    o, S_T = prefill(q, k, v, g, beta, S0)
    t1 = 9
    o1, S1 = prefill(q[:, :t1], k[:, :t1], v[:, :t1], g[:, :t1], beta[:, :t1], S0)
    o2, S2 = prefill(q[:, t1:], k[:, t1:], v[:, t1:], g[:, t1:], beta[:, t1:], S1.astype(np.float32))
    # S1 passes through fp32 between the two calls: compare with a matching tolerance
    return _rel(np.concatenate([o1, o2], 1), o) < 1e-6 and _rel(S2, S_T) < 1e-6 and \
        _rel(o1, o[:, :t1]) < RTOL


def pin_superposition(prefill):
    q, k, v1, g, beta, S01 = _case(seed=7)
    _, _, v2, _, _, S02 = _case(seed=8)
    oa, Sa = prefill(q, k, v1, g, beta, S01)
    ob, Sb = prefill(q, k, v2, g, beta, S02)
    # v1 + v2 and S01 + S02 are formed in float64 and are exact in float32 only approximately;
    # use inputs whose sum is exact: scale the second by a power of two.
    oc, Sc = prefill(q, k, (v1 + v2).astype(np.float32), g, beta, (S01 + S02).astype(np.float32))
    vsum = (v1 + v2).astype(np.float32).astype(np.float64)
    ok_inputs_exact = np.array_equal(vsum, v1.astype(np.float64) + v2.astype(np.float64))
    tol = RTOL if ok_inputs_exact else 1e-6
    return _rel(oc, oa + ob) < tol and _rel(Sc, Sa + Sb) < tol


def pin_row_permutation(prefill):
    q, k, v, g, beta, S0 = _case(seed=9)
    perm = np.random.default_rng(9).permutation(v.shape[-1])
    o, S_T = prefill(q, k, v, g, beta, S0)
    op, Sp = prefill(q, k, np.ascontiguousarray(v[..., perm]), g, beta,
                     np.ascontiguousarray(S0[:, :, perm, :]))
    return np.allclose(op, o[..., perm], rtol=0, atol=1e-13) and \
        np.allclose(Sp, S_T[:, :, perm, :], rtol=0, atol=1e-13)


def pin_padding_identity(prefill):
    q, k, v, g, beta, S0 = _case(T=11, seed=10)
    o, S_T = prefill(q, k, v, g, beta, S0)
    pad = 5
    rng = np.random.default_rng(10)
    qp = np.concatenate([q, rng.standard_normal(q[:, :pad].shape).astype(np.float32)], 1)
    kp = np.concatenate([k, np.zeros_like(k[:, :pad])], 1)
    vp = np.concatenate([v, rng.standard_normal(v[:, :pad].shape).astype(np.float32)], 1)
    gp = np.concatenate([g, np.zeros_like(g[:, :pad])], 1)
    bp = np.concatenate([beta, np.zeros_like(beta[:, :pad])], 1)
    o2, S2 = prefill(qp, kp, vp, gp, bp, S0)
    return np.array_equal(S2, S_T) and np.array_equal(o2[:, :11], o)


def pin_chain_independence(prefill):
    q, k, v, g, beta, S0 = _case(B=2, T=6, H=3, seed=11)
    o, S_T = prefill(q, k, v, g, beta, S0)
    for b in range(2):
        for h in range(3):
            o1, S1 = prefill(q[b:b + 1, :, h:h + 1], k[b:b + 1, :, h:h + 1], v[b:b + 1, :, h:h + 1],
                             g[b:b + 1, :, h:h + 1], beta[b:b + 1, :, h:h + 1],
                             S0[b:b + 1, h:h + 1])
            if not (np.array_equal(o1[0, :, 0], o[b, :, h]) and np.array_equal(S1[0, 0], S_T[b, h])):
                return False
    return True


PINS = [pin_beta0_g0_constant, pin_beta0_decay_closed_form, pin_beta1_writes_value,
        pin_brute_force, pin_exact_rational, pin_chunked_form, pin_split_carry,
        pin_superposition, pin_row_permutation, pin_padding_identity, pin_chain_independence]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_oracle_pin(pin):
    assert pin(oracle.prefill)


def test_decode_step_equals_prefill_t1():
    q, k, v, g, beta, S0 = _case(B=3, T=1, H=2, seed=12)
    o_p, S_p = oracle.prefill(q, k, v, g, beta, S0)
    o_d, S_d = oracle.decode_step(q[:, 0], k[:, 0], v[:, 0], g[:, 0], beta[:, 0], S0)
    assert np.array_equal(o_d, o_p[:, 0]) and np.array_equal(S_d, S_p)


def test_decode_steps_chain_equals_prefill():
    q, k, v, g, beta, S0 = _case(B=2, T=5, H=2, seed=13)
    o_p, S_p = oracle.prefill(q, k, v, g, beta, S0)
    S = S0.astype(np.float64)
    for t in range(5):
        o_d, S = oracle.decode_step(q[:, t], k[:, t], v[:, t], g[:, t], beta[:, t], S)
        assert _rel(o_d, o_p[:, t]) < 1e-15 or np.array_equal(o_d, o_p[:, t])
    assert np.array_equal(S, S_p)


def test_sampled_chains_match_full_run():
    q, k, v, g, beta, S0 = _case(B=2, T=9, H=3, seed=14)
    o, S_T = oracle.prefill(q, k, v, g, beta, S0)
    o2, S2 = oracle.prefill(q, k, v, g, beta, S0, chains=[1, 5])
    for c in (1, 5):
        b, h = divmod(c, 3)
        assert np.array_equal(o2[b, :, h], o[b, :, h]) and np.array_equal(S2[b, h], S_T[b, h])
    assert np.isnan(o2[0, :, 0]).all()


def test_full_head_dim_brute_force():
    """Head dim 128 (the pages' size) against the dense-product brute force, T = 4."""
    q, k, v, g, beta, S0 = _case(B=1, T=4, H=1, Dk=128, Dv=128, seed=15)
    o, S_T = oracle.prefill(q, k, v, g, beta, S0)
    ro, rS = _brute_force_chain(q[0, :, 0], k[0, :, 0], v[0, :, 0], g[0, :, 0], beta[0, :, 0], S0[0, 0])
    assert _rel(o[0, :, 0], ro) < 1e-11 and _rel(S_T[0, 0], rS) < 1e-11


# ----------------------------------------------------------------------------------------
# mutation check: each plausible mistake planted in a copy of the oracle fails some pin

MUTANTS = {
    "alpha_dropped_on_correction": ("Si[j] = alpha * Si[j] - alpha * bt * u[i] * kj",
                                    "Si[j] = alpha * Si[j] - bt * u[i] * kj"),
    "correction_sign_flipped": ("Si[j] = alpha * Si[j] - alpha * bt * u[i] * kj",
                                "Si[j] = alpha * Si[j] + alpha * bt * u[i] * kj"),
    "gate_not_applied_to_state": ("Si[j] = alpha * Si[j] - alpha", "Si[j] = Si[j] - alpha"),
    "alpha_from_negated_gate": ("const double alpha = exp(gt);", "const double alpha = exp(-gt);"),
    "beta_dropped_on_write": ("+ bt * vi * kj", "+ vi * kj"),
    "output_reads_key": ("for (int j = 0; j < Dk; ++j) acc += Si[j] * (double)qt[j];",
                         "for (int j = 0; j < Dk; ++j) acc += Si[j] * (double)kt[j];"),
    "transposed_state_read": ("for (int j = 0; j < Dk; ++j) acc += Si[j] * (double)kt[j];\n        u[i] = acc;",
                              "for (int j = 0; j < Dk; ++j) acc += S[(int64_t)(j % Dv) * Dk + (i % Dk)] * (double)kt[j];\n        u[i] = acc;"),
    "gate_of_head0_only": ("const int64_t gi = ((int64_t)b * T + t) * H + h;",
                           "const int64_t gi = ((int64_t)b * T + t) * H + 0;"),
    "initial_state_ignored": ("S[e] = (double)S0[s_off + e];", "S[e] = 0.0;"),
    "write_uses_k_for_v": ("const double vi = (double)vt[i];", "const double vi = (double)kt[i % Dk];"),
}


def _load_prefill_from(path):
    lib = ctypes.CDLL(path)
    fp = ctypes.POINTER(ctypes.c_float)
    dp = ctypes.POINTER(ctypes.c_double)
    lib.oracle_gdn_prefill_f64.argtypes = [fp] * 6 + [dp, dp] + [ctypes.c_int] * 5
    lib.oracle_gdn_prefill_f64.restype = ctypes.c_int

    def prefill(q, k, v, g, beta, S0=None):
        arrs = [np.ascontiguousarray(np.asarray(x, np.float32)) if x is not None else None
                for x in (q, k, v, g, beta, S0)]
        B, T, H, Dk = arrs[0].shape
        Dv = arrs[2].shape[-1]
        o = np.empty((B, T, H, Dv))
        S_T = np.empty((B, H, Dv, Dk))
        ptrs = [a.ctypes.data_as(fp) if a is not None else None for a in arrs]
        rc = lib.oracle_gdn_prefill_f64(*ptrs, o.ctypes.data_as(dp), S_T.ctypes.data_as(dp),
                                        B, T, H, Dk, Dv)
        assert rc == 0
        return o, S_T
    return prefill


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_every_planted_mistake_fails_a_pin(name):
    src_path = os.path.join(os.path.dirname(oracle.__file__), "gdn_oracle.c")
    src = open(src_path).read()
    old, new = MUTANTS[name]
    assert old in src, f"mutation anchor missing for {name}"
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "m.c")
        so = os.path.join(d, "m.so")
        open(c, "w").write(src.replace(old, new))
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-std=c99", "-o", so, c, "-lm"])
        prefill = _load_prefill_from(so)
        results = {p.__name__: bool(p(prefill)) for p in PINS}
    assert not all(results.values()), f"mutant {name} passed every pin: {results}"
