"""Seeded synthetic inputs for the gated delta rule.

This module is the ONE piece shared by the CUDA path's tests/benchmark and the
CPU oracle: it only draws random numbers and shapes them into the input
distribution the workloads use.  It holds none of the recurrence's arithmetic.

Recipe (per workload; all draws from ``numpy.random.default_rng(seed)`` on the
host, or a seeded ``torch.Generator`` on a CUDA device for the sizes too large
to draw on the host), in this order: q, k, v, g_raw, beta_raw, S0.

* q, k: N(0, 1) fp32 of shape [B, T, H, Dk], L2-normalised over Dk per (token,
  head) in fp32, then rounded to bf16 (round-to-nearest-even).
* v: N(0, 1) fp32 -> bf16.
* g = logsigmoid(g_raw) (evaluated in fp64, stored fp32), g_raw ~ N(g_mean, 1).
  alpha = exp(g) lies in (0, 1).
* beta = sigmoid(beta_raw) (fp64 -> fp32), beta_raw ~ N(0, 1).
* S0: zeros (None) or N(0, s0_std^2) fp32 of shape [B, H, Dv, Dk].

The workloads mirror the single-sequence, scalar-gate, head-dim-128 setting of
the ROCmFPX gated-delta-net prefill note (bittide.aicompass.dev article
d2880479, opening post: 512-token prefill calls) and add a batched decode
step and longer/larger prefills.  No public dataset is involved.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int
    Dk: int = 128
    Dv: int = 128
    g_mean: float = 0.0
    s0_std: Optional[float] = None
    decode_steps: int = 0          # > 0: a batched decode workload (T == 1 per step)
    chunks: tuple = (64,)

    @property
    def is_decode(self) -> bool:
        return self.decode_steps > 0

    def describe(self) -> str:
        if self.is_decode:
            return (f"decode B={self.B} H={self.H} Dk={self.Dk} Dv={self.Dv}, "
                    f"{self.decode_steps} steps, S~N(0,{self.s0_std}^2) fp32 in place")
        s0 = "S0=0" if self.s0_std is None else f"S0~N(0,{self.s0_std}^2)"
        return (f"prefill B={self.B} H={self.H} T={self.T} Dk={self.Dk} Dv={self.Dv}, "
                f"g=logsigmoid(N({self.g_mean},1)), beta=sigmoid(N(0,1)), {s0}")


WORKLOADS = {
    # small parity case the oracle finishes at once
    "tiny_b1_h2_t64": Workload("tiny_b1_h2_t64", B=1, H=2, T=64),
    # the pages' setting: one 512-token sequence, 16 heads; chunk 16 and 64 both timed
    "prefill_b1_h16_t512": Workload("prefill_b1_h16_t512", B=1, H=16, T=512, chunks=(64, 16)),
    # long prefill continuing from a carried state
    "prefill_b1_h16_t4096_s0": Workload("prefill_b1_h16_t4096_s0", B=1, H=16, T=4096, s0_std=0.02),
    # batched memory-bound decode: 64 sequences x 16 heads, 1 MiB of fp32 state per sequence
    "decode_b64_h16": Workload("decode_b64_h16", B=64, H=16, T=1, s0_std=0.02, decode_steps=256),
    # large batched prefill with long memory (alpha close to 1)
    "prefill_b4_h32_t32768": Workload("prefill_b4_h32_t32768", B=4, H=32, T=32768, g_mean=2.0),
}


def _logsigmoid64(x: np.ndarray) -> np.ndarray:
    return -np.logaddexp(0.0, -x.astype(np.float64))


def _sigmoid64(x: np.ndarray) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-x.astype(np.float64)))


def _l2norm_bf16_np(x: np.ndarray) -> torch.Tensor:
    n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True, dtype=np.float32)).astype(np.float32)
    return torch.from_numpy((x / n).astype(np.float32)).to(torch.bfloat16)


def prefill_inputs(B: int, T: int, H: int, Dk: int = 128, Dv: int = 128, *, seed: int = 0,
                   g_mean: float = 0.0, s0_std: Optional[float] = None,
                   device: str = "cpu") -> dict:
    """Draw one prefill batch.  Returns a dict of tensors on ``device``:
    q, k [B,T,H,Dk] bf16; v [B,T,H,Dv] bf16; g, beta [B,T,H] fp32;
    S0 [B,H,Dv,Dk] fp32 or None."""
    if str(device).startswith("cuda"):
        return _prefill_inputs_torch(B, T, H, Dk, Dv, seed, g_mean, s0_std, device)
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, H, Dk), dtype=np.float32)
    k = rng.standard_normal((B, T, H, Dk), dtype=np.float32)
    v = rng.standard_normal((B, T, H, Dv), dtype=np.float32)
    g_raw = rng.standard_normal((B, T, H), dtype=np.float32) + np.float32(g_mean)
    b_raw = rng.standard_normal((B, T, H), dtype=np.float32)
    S0 = None
    if s0_std is not None:
        S0 = torch.from_numpy((rng.standard_normal((B, H, Dv, Dk), dtype=np.float32)
                               * np.float32(s0_std)).astype(np.float32))
    return dict(q=_l2norm_bf16_np(q), k=_l2norm_bf16_np(k),
                v=torch.from_numpy(v).to(torch.bfloat16),
                g=torch.from_numpy(_logsigmoid64(g_raw).astype(np.float32)),
                beta=torch.from_numpy(_sigmoid64(b_raw).astype(np.float32)),
                S0=S0)


def _prefill_inputs_torch(B, T, H, Dk, Dv, seed, g_mean, s0_std, device):
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    out = {}
    for name, D in (("q", Dk), ("k", Dk)):
        x = torch.randn((B, T, H, D), generator=gen, device=device, dtype=torch.float32)
        x = x / torch.sqrt((x * x).sum(-1, keepdim=True))
        out[name] = x.to(torch.bfloat16)
        del x
    out["v"] = torch.randn((B, T, H, Dv), generator=gen, device=device,
                           dtype=torch.float32).to(torch.bfloat16)
    g_raw = torch.randn((B, T, H), generator=gen, device=device, dtype=torch.float64) + g_mean
    out["g"] = torch.nn.functional.logsigmoid(g_raw).to(torch.float32)
    b_raw = torch.randn((B, T, H), generator=gen, device=device, dtype=torch.float64)
    out["beta"] = torch.sigmoid(b_raw).to(torch.float32)
    out["S0"] = None
    if s0_std is not None:
        out["S0"] = torch.randn((B, H, Dv, Dk), generator=gen, device=device,
                                dtype=torch.float32) * s0_std
    return out


def kda_inputs(B: int, T: int, H: int, Dk: int = 128, Dv: int = 128, *, seed: int = 0,
               g_mean: float = 0.0, s0_std: Optional[float] = None,
               device: str = "cpu") -> dict:
    """Draw one batch for the per-channel gate (KDA).  The recipe of
    ``prefill_inputs`` with one gate draw per key channel: g [B,T,H,Dk] fp32 =
    logsigmoid(N(g_mean, 1)).  Draw order q, k, v, g_raw, beta_raw, S0."""
    if str(device).startswith("cuda"):
        gen = torch.Generator(device=device)
        gen.manual_seed(seed)
        out = {}
        for name, D in (("q", Dk), ("k", Dk)):
            x = torch.randn((B, T, H, D), generator=gen, device=device, dtype=torch.float32)
            out[name] = (x / torch.sqrt((x * x).sum(-1, keepdim=True))).to(torch.bfloat16)
            del x
        out["v"] = torch.randn((B, T, H, Dv), generator=gen, device=device,
                               dtype=torch.float32).to(torch.bfloat16)
        g_raw = torch.randn((B, T, H, Dk), generator=gen, device=device,
                            dtype=torch.float64) + g_mean
        out["g"] = torch.nn.functional.logsigmoid(g_raw).to(torch.float32)
        del g_raw
        b_raw = torch.randn((B, T, H), generator=gen, device=device, dtype=torch.float64)
        out["beta"] = torch.sigmoid(b_raw).to(torch.float32)
        out["S0"] = None
        if s0_std is not None:
            out["S0"] = torch.randn((B, H, Dv, Dk), generator=gen, device=device,
                                    dtype=torch.float32) * s0_std
        return out
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, H, Dk), dtype=np.float32)
    k = rng.standard_normal((B, T, H, Dk), dtype=np.float32)
    v = rng.standard_normal((B, T, H, Dv), dtype=np.float32)
    g_raw = rng.standard_normal((B, T, H, Dk), dtype=np.float32) + np.float32(g_mean)
    b_raw = rng.standard_normal((B, T, H), dtype=np.float32)
    S0 = None
    if s0_std is not None:
        S0 = torch.from_numpy((rng.standard_normal((B, H, Dv, Dk), dtype=np.float32)
                               * np.float32(s0_std)).astype(np.float32))
    return dict(q=_l2norm_bf16_np(q), k=_l2norm_bf16_np(k),
                v=torch.from_numpy(v).to(torch.bfloat16),
                g=torch.from_numpy(_logsigmoid64(g_raw).astype(np.float32)),
                beta=torch.from_numpy(_sigmoid64(b_raw).astype(np.float32)),
                S0=S0)


def decode_inputs(B: int, H: int, steps: int, Dk: int = 128, Dv: int = 128, *, seed: int = 0,
                  g_mean: float = 0.0, s0_std: float = 0.02, device: str = "cpu") -> dict:
    """Draw ``steps`` decode steps up front.  q, k [steps,B,H,Dk] bf16;
    v [steps,B,H,Dv] bf16; g, beta [steps,B,H] fp32; S [B,H,Dv,Dk] fp32."""
    d = prefill_inputs(B, steps, H, Dk, Dv, seed=seed, g_mean=g_mean, s0_std=s0_std,
                       device=device)
    # [B, steps, H, D] -> [steps, B, H, D]
    return dict(q=d["q"].transpose(0, 1).contiguous(), k=d["k"].transpose(0, 1).contiguous(),
                v=d["v"].transpose(0, 1).contiguous(), g=d["g"].transpose(0, 1).contiguous(),
                beta=d["beta"].transpose(0, 1).contiguous(), S=d["S0"])


def workload_inputs(w: Workload, *, seed: int = 0, device: str = "cpu") -> dict:
    if w.is_decode:
        return decode_inputs(w.B, w.H, w.decode_steps, w.Dk, w.Dv, seed=seed, g_mean=w.g_mean,
                             s0_std=w.s0_std if w.s0_std is not None else 0.0, device=device)
    return prefill_inputs(w.B, w.T, w.H, w.Dk, w.Dv, seed=seed, g_mean=w.g_mean,
                          s0_std=w.s0_std, device=device)
