"""Gated delta rule (gated DeltaNet) prefill and decode for NVIDIA B200 (sm_100a).

The compute lives in ``libgdn_b200.so`` (hand-written CUDA, C ABI declared in
``include/gdn.h``); ``gdn.py`` is a thin ctypes binding that only marshals
torch tensors and the current CUDA stream into that ABI.  There is no CPU
fallback: calling into the binding without the built library raises.

    from gated_deltanet_linear_20_b200 import prefill, decode_step, kda_prefill
    o, S_T = prefill(q, k, v, g, beta, S0=None, chunk=64)
    o = decode_step(q, k, v, g, beta, S)       # S updated in place
    o, S_T = kda_prefill(q, k, v, g_vec, beta)  # per-channel gate: g_vec [B,T,H,Dk]

Head dims 64, 128 and 256 (Dk != Dv allowed) are accepted.  Prefill with
Dk = 64 or 128 runs the chunked tensor-core kernel, with Dk = 256 the
row-parallel fp32 kernel; the per-channel-gate prefill runs its own chunked
tensor-core kernel with Dk = 128 (any Dv); decode at 128 x 128 and 64 x 64 streams the
state through the decode kernels, at other dims through the row kernel.

The binding is imported lazily so that ``inputs`` (the seeded input
generator) can be used without loading the CUDA library.
"""
from __future__ import annotations

__all__ = ["prefill", "decode_step", "decode_tokens", "prefill_varlen", "kda_prefill",
           "kda_prefill_varlen", "kda_decode", "abi_version", "status_str", "query_status",
           "GDNError"]


def __getattr__(name):
    if name in ("prefill", "decode_step", "decode_tokens", "prefill_varlen", "kda_prefill",
                "kda_prefill_varlen", "kda_decode", "abi_version", "status_str", "query_status", "GDNError",
                "library_path"):
        import importlib
        return getattr(importlib.import_module(__name__ + ".gdn"), name)
    raise AttributeError(name)
