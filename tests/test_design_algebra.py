"""CPU checks of the two regroupings of the recurrence that the kernels rely
on, each restated here in fp64 numpy and compared with the oracle:

* the segmented schedule: over a stretch of tokens the state is affine in the
  state the stretch starts from, S_t = S_k F_{k,t} + R_{k,t} and
  o_t = S_k (F_{k,t} q_t) + o^R_t, where F is the state reached from the
  identity with v = 0 and R, o^R the state and output from zero;
* the token pairs of the row-parallel kernel: with s' = alpha_t o s and
  u = alpha_{t+1} o s', the second token's residual and output follow from
  u.k_{t+1}, u.q_{t+1} and the token-only scalars c = (k_t o alpha_{t+1}).k_{t+1}
  and e = (k_t o alpha_{t+1}).q_{t+1}.
"""
from __future__ import annotations

import numpy as np

import oracle


def _chain(seed, T, Dk, Dv, vector_gate):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, Dk))
    k = rng.standard_normal((T, Dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, Dv))
    g = -rng.uniform(0.01, 1.0, (T, Dk) if vector_gate else (T,))
    beta = rng.uniform(0.0, 1.0, T)
    S0 = 0.3 * rng.standard_normal((Dv, Dk))
    return [x.astype(np.float32) for x in (q, k, v, g, beta, S0)]


def _run(q, k, v, g, beta, S0, vector_gate):
    f = oracle.kda_prefill if vector_gate else oracle.prefill
    o, S = f(q[None, :, None], k[None, :, None], v[None, :, None], g[None, :, None],
             beta[None, :, None], None if S0 is None else S0[None, None])
    return o[0, :, 0], S[0, 0]


def _rel(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def test_segment_decomposition_matches_the_oracle():
    """Four segments run from zero (R) and from the identity with v = 0 (F),
    then chained S_{k+1} = S_k F_k + R_k and o_t += S_k f_t, equal the
    single pass."""
    T, Dk, Dv, nseg = 40, 8, 6, 4
    q, k, v, g, beta, S0 = _chain(1, T, Dk, Dv, False)
    o_ref, S_ref = _run(q, k, v, g, beta, S0, False)
    L = T // nseg
    S = S0.astype(np.float64)
    o = np.zeros((T, Dv))
    for s in range(nseg):
        sl = slice(s * L, (s + 1) * L)
        oR, R = _run(q[sl], k[sl], v[sl], g[sl], beta[sl], None, False)
        # F (Dk x Dk): the same stretch from the identity, with v = 0
        eye = np.eye(Dk, dtype=np.float32)
        zero_v = np.zeros((L, Dk), np.float32)
        f_t, F = _run(q[sl], k[sl], zero_v, g[sl], beta[sl], eye, False)
        o[sl] = oR + f_t @ S.T          # o_t = o^R_t + S_k (F_t q_t)
        S = S @ F + R                    # S_{k+1} = S_k F_k + R_k
    assert _rel(o, o_ref) < 1e-10 and _rel(S, S_ref) < 1e-10


def _pairs(q, k, v, g, beta, S0, vector_gate):
    """The row kernel's pairwise update, row by row, in fp64."""
    q, k, v, g, beta, S = (x.astype(np.float64) for x in (q, k, v, g, beta, S0))
    T, Dk = k.shape
    a = np.exp(g) if vector_gate else np.exp(g)[:, None] * np.ones(Dk)
    o = np.zeros((T, S.shape[0]))
    t = 0
    while t + 1 < T:
        sp = S * a[t]                   # s' = s o alpha_t (every row)
        u = sp * a[t + 1]
        ka = k[t] * a[t + 1]
        c, e = ka @ k[t + 1], ka @ q[t + 1]
        x0, y0, x1, y1 = sp @ k[t], sp @ q[t], u @ k[t + 1], u @ q[t + 1]
        d0 = beta[t] * (v[t] - x0)
        d1 = beta[t + 1] * (v[t + 1] - (x1 + d0 * c))
        o[t] = y0 + d0 * (k[t] @ q[t])
        o[t + 1] = y1 + d0 * e + d1 * (k[t + 1] @ q[t + 1])
        S = u + np.outer(d0, ka) + np.outer(d1, k[t + 1])
        t += 2
    if t < T:                           # a last odd token: the one-token step
        sp = S * a[t]
        d = beta[t] * (v[t] - sp @ k[t])
        S = sp + np.outer(d, k[t])
        o[t] = S @ q[t]
    return o, S


def test_token_pairs_match_the_oracle():
    for vector_gate in (False, True):
        for T in (10, 11):
            q, k, v, g, beta, S0 = _chain(2 + T, T, 16, 12, vector_gate)
            o_ref, S_ref = _run(q, k, v, g, beta, S0, vector_gate)
            o, S = _pairs(q, k, v, g, beta, S0, vector_gate)
            assert _rel(o, o_ref) < 1e-11 and _rel(S, S_ref) < 1e-11, (vector_gate, T)
