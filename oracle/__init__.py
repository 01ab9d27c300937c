"""fp64 CPU oracle for the gated delta rule -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The
product path (``gated_deltanet_linear_20_b200``) never imports, links or runs
it, and the two share no code: the only thing both sides consume is the seeded
input generator, which holds none of the method's arithmetic.

What is computed (per sequence b and head h, independently), in fp64:

    alpha_t = exp(g_t)
    S_t     = alpha_t * S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
    o_t     = S_t q_t

This is the gated delta rule of the hybrid Qwen 3.5 linear-attention layers.
``kda_prefill`` is the per-channel-gate variant (KDA): alpha_t becomes a vector
over Dk, applied as S_{t-1} diag(alpha_t) in place of alpha_t S_{t-1}.
The ROCmFPX gated-delta-net prefill note (bittide.aicompass.dev article
d2880479, opening post) fixes its setting -- scalar gate per token and head,
head dim 128, single-sequence prefill, state in F32 accumulators -- but prints
no formula and no worked example, so this file is pinned by the invariants and
brute-force checks in ``tests/test_oracle_pins.py`` rather than by printed
values.  The arithmetic lives in ``gdn_oracle.c`` (plain C, no fast-math,
OpenMP over the B*H independent chains); this module only marshals arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libgdn_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile gdn_oracle.c with gcc (-O2, no fast-math, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        fp = ctypes.POINTER(ctypes.c_float)
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int)
        ci = ctypes.c_int
        lib.oracle_gdn_prefill_f64.argtypes = [fp, fp, fp, fp, fp, fp, dp, dp, ci, ci, ci, ci, ci]
        lib.oracle_gdn_prefill_f64.restype = ci
        lib.oracle_gdn_prefill_chains_f64.argtypes = [fp, fp, fp, fp, fp, fp, dp, dp,
                                                      ci, ci, ci, ci, ci, ip, ci]
        lib.oracle_gdn_prefill_chains_f64.restype = ci
        lib.oracle_gdn_decode_step_f64.argtypes = [fp, fp, fp, fp, fp, dp, dp, ci, ci, ci, ci]
        lib.oracle_gdn_decode_step_f64.restype = ci
        lib.oracle_kda_prefill_f64.argtypes = [fp, fp, fp, fp, fp, fp, dp, dp, ci, ci, ci, ci, ci]
        lib.oracle_kda_prefill_f64.restype = ci
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = ci
        _lib = lib
    return _lib


def _f32(x):
    """Widen to a contiguous float32 numpy array (exact for bf16 inputs)."""
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor
        x = x.detach().to("cpu")
        import torch
        x = x.to(torch.float32).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


def _ptr(a, ctype):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def num_threads() -> int:
    """OpenMP threads the oracle uses."""
    return int(_load().oracle_num_threads())


def prefill(q, k, v, g, beta, S0=None, chains=None):
    """Run the recurrence over all T tokens.

    q, k: [B,T,H,Dk]; v: [B,T,H,Dv]; g, beta: [B,T,H]; S0: [B,H,Dv,Dk] or None.
    Returns (o [B,T,H,Dv], S_T [B,H,Dv,Dk]) as float64 numpy arrays.  With
    ``chains`` (an iterable of b*H+h ids) only those chains are computed; the
    other entries of the outputs are NaN.
    """
    q, k, v, g, beta, S0 = (_f32(t) for t in (q, k, v, g, beta, S0))
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    assert k.shape == (B, T, H, Dk) and v.shape == (B, T, H, Dv)
    assert g.shape == (B, T, H) and beta.shape == (B, T, H)
    assert S0 is None or S0.shape == (B, H, Dv, Dk)
    lib = _load()
    if chains is None:
        o = np.empty((B, T, H, Dv), np.float64)
        S_T = np.empty((B, H, Dv, Dk), np.float64)
        rc = lib.oracle_gdn_prefill_f64(_ptr(q, ctypes.c_float), _ptr(k, ctypes.c_float),
                                        _ptr(v, ctypes.c_float), _ptr(g, ctypes.c_float),
                                        _ptr(beta, ctypes.c_float), _ptr(S0, ctypes.c_float),
                                        _ptr(o, ctypes.c_double), _ptr(S_T, ctypes.c_double),
                                        B, T, H, Dk, Dv)
    else:
        ids = np.ascontiguousarray(np.asarray(list(chains), dtype=np.int32))
        o = np.full((B, T, H, Dv), np.nan, np.float64)
        S_T = np.full((B, H, Dv, Dk), np.nan, np.float64)
        rc = lib.oracle_gdn_prefill_chains_f64(_ptr(q, ctypes.c_float), _ptr(k, ctypes.c_float),
                                               _ptr(v, ctypes.c_float), _ptr(g, ctypes.c_float),
                                               _ptr(beta, ctypes.c_float), _ptr(S0, ctypes.c_float),
                                               _ptr(o, ctypes.c_double), _ptr(S_T, ctypes.c_double),
                                               B, T, H, Dk, Dv, _ptr(ids, ctypes.c_int), len(ids))
    if rc != 0:
        raise RuntimeError(f"oracle prefill failed with code {rc}")
    return o, S_T


def decode_step(q, k, v, g, beta, S):
    """One decode step: q, k [B,H,Dk]; v [B,H,Dv]; g, beta [B,H]; S [B,H,Dv,Dk].

    Returns (o [B,H,Dv], S_new [B,H,Dv,Dk]) in float64; the input S is not
    modified (it is copied to a float64 state first).
    """
    q, k, v, g, beta = (_f32(t) for t in (q, k, v, g, beta))
    if hasattr(S, "detach"):
        S = S.detach().to("cpu").double().numpy()
    S = np.array(S, dtype=np.float64, order="C", copy=True)
    B, H, Dk = q.shape
    Dv = v.shape[-1]
    assert S.shape == (B, H, Dv, Dk) and g.shape == (B, H) and beta.shape == (B, H)
    o = np.empty((B, H, Dv), np.float64)
    rc = _load().oracle_gdn_decode_step_f64(_ptr(q, ctypes.c_float), _ptr(k, ctypes.c_float),
                                            _ptr(v, ctypes.c_float), _ptr(g, ctypes.c_float),
                                            _ptr(beta, ctypes.c_float), _ptr(S, ctypes.c_double),
                                            _ptr(o, ctypes.c_double), B, H, Dk, Dv)
    if rc != 0:
        raise RuntimeError(f"oracle decode failed with code {rc}")
    return o, S


def kda_prefill(q, k, v, g, beta, S0=None):
    """Per-channel gate (KDA): alpha_t = exp(g_t) over Dk,
    S_t = S_{t-1} diag(alpha_t)(I - beta_t k_t k_t^T) + beta_t v_t k_t^T, o_t = S_t q_t.

    q, k: [B,T,H,Dk]; v: [B,T,H,Dv]; g: [B,T,H,Dk]; beta: [B,T,H]; S0: [B,H,Dv,Dk]
    or None.  Returns (o [B,T,H,Dv], S_T [B,H,Dv,Dk]) as float64 numpy arrays.
    """
    q, k, v, g, beta, S0 = (_f32(t) for t in (q, k, v, g, beta, S0))
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    assert k.shape == (B, T, H, Dk) and v.shape == (B, T, H, Dv)
    assert g.shape == (B, T, H, Dk) and beta.shape == (B, T, H)
    assert S0 is None or S0.shape == (B, H, Dv, Dk)
    o = np.empty((B, T, H, Dv), np.float64)
    S_T = np.empty((B, H, Dv, Dk), np.float64)
    rc = _load().oracle_kda_prefill_f64(_ptr(q, ctypes.c_float), _ptr(k, ctypes.c_float),
                                        _ptr(v, ctypes.c_float), _ptr(g, ctypes.c_float),
                                        _ptr(beta, ctypes.c_float), _ptr(S0, ctypes.c_float),
                                        _ptr(o, ctypes.c_double), _ptr(S_T, ctypes.c_double),
                                        B, T, H, Dk, Dv)
    if rc != 0:
        raise RuntimeError(f"oracle KDA prefill failed with code {rc}")
    return o, S_T
