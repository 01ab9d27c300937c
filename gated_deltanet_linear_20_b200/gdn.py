"""ctypes binding of libgdn_b200.so (C ABI in include/gdn.h).

Argument marshalling only: checks dtypes, shapes, devices and contiguity,
allocates outputs with torch, and passes raw device pointers plus the current
CUDA stream to the library.  Every step of the computation runs in the
library's CUDA kernels; there is no fallback.  Importing this module without
the built library raises ImportError.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libgdn_b200.so")

if not os.path.exists(library_path):
    raise ImportError(f"{library_path} is missing: build it with "
                      "`python -m gated_deltanet_linear_20_b200.build` (nvcc, sm_100a)")

_lib = ctypes.CDLL(library_path)
_vp, _ci = ctypes.c_void_p, ctypes.c_int
_lib.gdn_abi_version.argtypes = []
_lib.gdn_abi_version.restype = _ci
_lib.gdn_status_str.argtypes = [_ci]
_lib.gdn_status_str.restype = ctypes.c_char_p
_lib.gdn_prefill.argtypes = [_vp] * 8 + [_ci] * 6 + [_vp, _vp]
_lib.gdn_prefill.restype = _ci
_lib.gdn_prefill_workspace_bytes.argtypes = [_ci] * 6
_lib.gdn_prefill_workspace_bytes.restype = ctypes.c_size_t
_lib.gdn_prefill_ws.argtypes = [_vp] * 8 + [_ci] * 6 + [_vp, ctypes.c_size_t, _vp, _vp]
_lib.gdn_prefill_ws.restype = _ci
_lib.gdn_prefill_varlen.argtypes = [_vp] * 9 + [_ci] * 6 + [_vp, _ci, _ci, _vp, _vp]
_lib.gdn_prefill_varlen.restype = _ci
class Options(ctypes.Structure):
    """gdn_options (include/gdn.h)."""
    _fields_ = [("size", ctypes.c_int), ("qk_l2norm", ctypes.c_int), ("q_scale", ctypes.c_float),
                ("o_bf16", ctypes.c_int)]


def _options(qk_l2norm: bool, q_scale: float, o_bf16: bool = False):
    if not qk_l2norm and q_scale == 1.0 and not o_bf16:
        return None
    return ctypes.byref(Options(ctypes.sizeof(Options), int(bool(qk_l2norm)), float(q_scale),
                                int(bool(o_bf16))))


_lib.gdn_prefill_ex.argtypes = [_vp] * 8 + [_ci] * 6 + [_vp, ctypes.c_size_t, _vp, _vp, _vp]
_lib.gdn_prefill_ex.restype = _ci
_lib.gdn_decode_ex.argtypes = [_vp] * 7 + [_ci] * 5 + [_vp, _vp, _vp]
_lib.gdn_decode_ex.restype = _ci
_lib.gdn_prefill_static_ws.argtypes = [_vp] * 8 + [_ci] * 6 + [_vp, _vp]
_lib.gdn_prefill_static_ws.restype = _ci
_lib.gdn_prefill_schedule.argtypes = [_ci] * 4 + [_vp, _vp, _vp]
_lib.gdn_prefill_schedule.restype = _ci
_lib.gdn_decode_step.argtypes = [_vp] * 7 + [_ci] * 4 + [_vp, _vp]
_lib.gdn_decode_step.restype = _ci
_lib.gdn_decode_tokens.argtypes = [_vp] * 7 + [_ci] * 5 + [_vp, _vp]
_lib.gdn_decode_tokens.restype = _ci
_lib.gdn_kda_prefill.argtypes = [_vp] * 8 + [_ci] * 5 + [_vp, _vp]
_lib.gdn_kda_prefill.restype = _ci
_lib.gdn_kda_decode.argtypes = [_vp] * 7 + [_ci] * 5 + [_vp, _vp]
_lib.gdn_kda_decode.restype = _ci
_lib.gdn_kda_prefill_ex.argtypes = [_vp] * 8 + [_ci] * 5 + [_vp, _vp, _vp]
_lib.gdn_kda_prefill_ex.restype = _ci
_lib.gdn_kda_decode_ex.argtypes = [_vp] * 7 + [_ci] * 5 + [_vp, _vp, _vp]
_lib.gdn_kda_decode_ex.restype = _ci
_lib.gdn_kda_prefill_varlen.argtypes = [_vp] * 9 + [_ci] * 5 + [_vp, _ci, _ci, _vp, _vp]
_lib.gdn_kda_prefill_varlen.restype = _ci
_lib.gdn_prefill_varlen_ex.argtypes = [_vp] * 9 + [_ci] * 6 + [_vp, _ci, _ci, _vp, _vp, _vp]
_lib.gdn_prefill_varlen_ex.restype = _ci
_lib.gdn_kda_prefill_varlen_ex.argtypes = [_vp] * 9 + [_ci] * 5 + [_vp, _ci, _ci, _vp, _vp, _vp]
_lib.gdn_kda_prefill_varlen_ex.restype = _ci
_lib.gdn_query_status.argtypes = [_vp, _vp]
_lib.gdn_query_status.restype = _ci

ABI_VERSION = 8
if _lib.gdn_abi_version() != ABI_VERSION:
    raise ImportError(f"libgdn_b200.so ABI {_lib.gdn_abi_version()} != binding ABI {ABI_VERSION}")

# status codes (include/gdn.h)
GDN_OK = 0
GDN_ERR_NULL = -1
GDN_ERR_ALIGN = -2
GDN_ERR_SHAPE = -3
GDN_ERR_UNSUPPORTED = -4
GDN_ERR_ALIAS = -5
GDN_ERR_LAUNCH = -6
GDN_ERR_DEVICE_TIMEOUT = -7
GDN_ERR_WORKSPACE = -8
GDN_ERR_STATIC_WORKSPACE_LIMIT = -9
STATIC_WORKSPACE_BYTES = 16 << 20  # GDN_STATIC_WORKSPACE_BYTES


class GDNError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_str(code)} (code {code})")


def abi_version() -> int:
    return int(_lib.gdn_abi_version())


def status_str(code: int) -> str:
    return _lib.gdn_status_str(int(code)).decode()


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(device: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _check(t: torch.Tensor, name: str, dtype: torch.dtype, shape: tuple, device):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def workspace_bytes(B: int, T: int, H: int, chunk: int = 64, Dk: int = 128, Dv: int = 128) -> int:
    """Bytes of workspace gdn_prefill_ws needs on the current device (0: single pass)."""
    return int(_lib.gdn_prefill_workspace_bytes(B, T, H, Dk, Dv, int(chunk)))


def schedule(B: int, T: int, H: int, num_sms: int) -> Tuple[int, int, int]:
    """(segments per chain, tiles per segment, workspace bytes) that gdn_prefill_ws
    picks on a device with ``num_sms`` multiprocessors."""
    n, L, ws = ctypes.c_int(), ctypes.c_int(), ctypes.c_size_t()
    rc = _lib.gdn_prefill_schedule(B, T, H, num_sms, ctypes.byref(n), ctypes.byref(L),
                                   ctypes.byref(ws))
    if rc != GDN_OK:
        raise GDNError(rc, "gdn_prefill_schedule")
    return n.value, L.value, ws.value


def prefill(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor,
            beta: torch.Tensor, S0: Optional[torch.Tensor] = None, chunk: int = 64, *,
            o: Optional[torch.Tensor] = None, S_T: Optional[torch.Tensor] = None,
            status: Optional[torch.Tensor] = None, segmented: bool = True,
            workspace: Optional[torch.Tensor] = None, qk_l2norm: bool = False,
            q_scale: float = 1.0, o_bf16: bool = False) -> Tuple[torch.Tensor, torch.Tensor]:
    """Chunked prefill: returns (o [B,T,H,Dv] fp32 or bf16, S_T [B,H,Dv,Dk] fp32).

    q, k [B,T,H,Dk] bf16; v [B,T,H,Dv] bf16; g, beta [B,T,H] fp32; S0 [B,H,Dv,Dk]
    fp32 or None (zeros); chunk 16 or 64.  Launches on the current stream.
    ``o`` / ``S_T`` may be given preallocated (``S_T`` may be ``S0``).
    ``segmented`` calls gdn_prefill_ws, which cuts chains into segments walked
    in parallel when they are too few to fill the GPU; its workspace is
    ``workspace`` (a uint8 CUDA tensor) or a fresh torch allocation.  With
    ``segmented=False`` it calls gdn_prefill (one pass per chain).
    ``qk_l2norm`` / ``q_scale`` (gdn_options) normalise q and k per token and
    head and scale q inside the kernel (gdn_prefill_ex).  ``o_bf16`` makes o
    bf16 (the fp32 value rounded to nearest even); it runs the single pass.
    Dk, Dv may each be 64, 128 or 256.  With Dk = 64 or 128 the chunked
    tensor-core kernel runs (Dv = 256 on two CTAs per chain); with Dk = 256 the
    row-parallel fp32 kernel.  Segments apply at 128 x 128 only; the fused
    options on the tensor-core kernel (not with Dk = 256)."""
    if q.dim() != 4:
        raise ValueError("q must be [B,T,H,Dk]")
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("gdn.prefill runs on CUDA tensors only (no CPU path)")
    _check(q, "q", torch.bfloat16, (B, T, H, Dk), dev)
    _check(k, "k", torch.bfloat16, (B, T, H, Dk), dev)
    _check(v, "v", torch.bfloat16, (B, T, H, Dv), dev)
    _check(g, "g", torch.float32, (B, T, H), dev)
    _check(beta, "beta", torch.float32, (B, T, H), dev)
    if S0 is not None:
        _check(S0, "S0", torch.float32, (B, H, Dv, Dk), dev)
    o_dtype = torch.bfloat16 if o_bf16 else torch.float32
    if o is None:
        o = torch.empty((B, T, H, Dv), dtype=o_dtype, device=dev)
    _check(o, "o", o_dtype, (B, T, H, Dv), dev)
    if S_T is None:
        S_T = torch.empty((B, H, Dv, Dk), dtype=torch.float32, device=dev)
    _check(S_T, "S_T", torch.float32, (B, H, Dv, Dk), dev)
    if status is not None:
        _check(status, "status", torch.int32, (1,), dev)
    opts = _options(qk_l2norm, q_scale, o_bf16)
    if not segmented or o_bf16:
        if opts is None:
            rc = _lib.gdn_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0),
                                  _ptr(o), _ptr(S_T), B, T, H, Dk, Dv, int(chunk), _ptr(status),
                                  _stream_handle(dev))
        else:
            rc = _lib.gdn_prefill_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0),
                                     _ptr(o), _ptr(S_T), B, T, H, Dk, Dv, int(chunk), None,
                                     ctypes.c_size_t(0), opts, _ptr(status), _stream_handle(dev))
        if rc != GDN_OK:
            raise GDNError(rc, "gdn_prefill")
        return o, S_T
    if workspace is None:
        with torch.cuda.device(dev):
            need = workspace_bytes(B, T, H, chunk, Dk, Dv)
        if need > 0:
            workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    if workspace is not None:
        if workspace.dtype != torch.uint8 or workspace.device != dev or not workspace.is_contiguous():
            raise ValueError("workspace must be a contiguous uint8 tensor on the inputs' device")
    ws_bytes = 0 if workspace is None else workspace.numel()
    if opts is None:
        rc = _lib.gdn_prefill_ws(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0), _ptr(o),
                                 _ptr(S_T), B, T, H, Dk, Dv, int(chunk), _ptr(workspace),
                                 ctypes.c_size_t(ws_bytes), _ptr(status), _stream_handle(dev))
    else:
        # workspace is None only when the schedule is the single pass, which is
        # what gdn_prefill_ex runs for a NULL workspace
        rc = _lib.gdn_prefill_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0), _ptr(o),
                                 _ptr(S_T), B, T, H, Dk, Dv, int(chunk), _ptr(workspace),
                                 ctypes.c_size_t(ws_bytes), opts, _ptr(status), _stream_handle(dev))
    if rc != GDN_OK:
        raise GDNError(rc, "gdn_prefill_ws")
    return o, S_T


def prefill_varlen(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor,
                   beta: torch.Tensor, cu_seqlens: torch.Tensor, S0: Optional[torch.Tensor] = None,
                   chunk: int = 64, *, o: Optional[torch.Tensor] = None,
                   S_T: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
                   snap_every: int = 0,
                   snaps: Optional[torch.Tensor] = None, qk_l2norm: bool = False,
                   q_scale: float = 1.0, o_bf16: bool = False):
    """Prefill of N packed sequences: q, k [total_T,H,Dk] bf16; v [total_T,H,Dv] bf16;
    g, beta [total_T,H] fp32; cu_seqlens int32 [N+1] on the device (offsets of
    the sequences).  Returns (o [total_T,H,Dv] fp32, S_T [N,H,Dv,Dk] fp32).
    With ``snap_every`` (a multiple of 64) it also returns the state snapshots
    [n_snaps,H,Dv,Dk] (after every snap_every tokens of each sequence, sequence
    by sequence); ``snaps`` may be given preallocated, else its size is read
    from cu_seqlens (one device-to-host copy).  Dk 64 or 128, Dv 64, 128 or
    256 (the chunked tensor-core kernel).  ``qk_l2norm`` / ``q_scale`` apply the
    fused pre-steps of ``prefill`` and ``o_bf16`` writes o as bf16
    (gdn_prefill_varlen_ex)."""
    if q.dim() != 3:
        raise ValueError("q must be [total_T,H,Dk]")
    total_T, H, Dk = q.shape
    Dv = v.shape[-1]
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("gdn.prefill_varlen runs on CUDA tensors only (no CPU path)")
    if cu_seqlens.dim() != 1 or cu_seqlens.numel() < 1:
        raise ValueError("cu_seqlens must be [N+1]")
    N = cu_seqlens.numel() - 1
    _check(cu_seqlens, "cu_seqlens", torch.int32, (N + 1,), dev)
    _check(q, "q", torch.bfloat16, (total_T, H, Dk), dev)
    _check(k, "k", torch.bfloat16, (total_T, H, Dk), dev)
    _check(v, "v", torch.bfloat16, (total_T, H, Dv), dev)
    _check(g, "g", torch.float32, (total_T, H), dev)
    _check(beta, "beta", torch.float32, (total_T, H), dev)
    if S0 is not None:
        _check(S0, "S0", torch.float32, (N, H, Dv, Dk), dev)
    o_dtype = torch.bfloat16 if o_bf16 else torch.float32
    if o is None:
        o = torch.empty((total_T, H, Dv), dtype=o_dtype, device=dev)
    _check(o, "o", o_dtype, (total_T, H, Dv), dev)
    if S_T is None:
        S_T = torch.empty((N, H, Dv, Dk), dtype=torch.float32, device=dev)
    _check(S_T, "S_T", torch.float32, (N, H, Dv, Dk), dev)
    if status is not None:
        _check(status, "status", torch.int32, (1,), dev)
    n_snaps = 0
    if snap_every:
        if snaps is None:
            lens = (cu_seqlens[1:] - cu_seqlens[:-1]).cpu()
            n_snaps = int((lens // int(snap_every)).sum())
            snaps = torch.empty((n_snaps, H, Dv, Dk), dtype=torch.float32, device=dev)
        n_snaps = snaps.shape[0]
        _check(snaps, "snaps", torch.float32, (n_snaps, H, Dv, Dk), dev)
    else:
        snaps = None
    opts = _options(qk_l2norm, q_scale, o_bf16)
    if opts is None:
        rc = _lib.gdn_prefill_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0),
                                     _ptr(o), _ptr(S_T), _ptr(cu_seqlens), N, total_T, H, Dk, Dv,
                                     int(chunk), _ptr(snaps), int(snap_every), n_snaps,
                                     _ptr(status), _stream_handle(dev))
    else:
        rc = _lib.gdn_prefill_varlen_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0),
                                        _ptr(o), _ptr(S_T), _ptr(cu_seqlens), N, total_T, H, Dk,
                                        Dv, int(chunk), _ptr(snaps), int(snap_every), n_snaps,
                                        opts, _ptr(status), _stream_handle(dev))
    if rc != GDN_OK:
        raise GDNError(rc, "gdn_prefill_varlen")
    return (o, S_T) if snaps is None else (o, S_T, snaps)


def prefill_static(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor,
                   beta: torch.Tensor, S0: Optional[torch.Tensor] = None, chunk: int = 64, *,
                   o: Optional[torch.Tensor] = None, S_T: Optional[torch.Tensor] = None,
                   status: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """gdn_prefill_static_ws: the segmented schedule on the library's built-in
    16 MiB device scratch (no allocation).  Calls that may overlap on a device
    race on that scratch; larger problems raise GDNError(GDN_ERR_STATIC_WORKSPACE_LIMIT)."""
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("gdn.prefill_static runs on CUDA tensors only (no CPU path)")
    _check(q, "q", torch.bfloat16, (B, T, H, Dk), dev)
    _check(k, "k", torch.bfloat16, (B, T, H, Dk), dev)
    _check(v, "v", torch.bfloat16, (B, T, H, Dv), dev)
    _check(g, "g", torch.float32, (B, T, H), dev)
    _check(beta, "beta", torch.float32, (B, T, H), dev)
    if S0 is not None:
        _check(S0, "S0", torch.float32, (B, H, Dv, Dk), dev)
    if o is None:
        o = torch.empty((B, T, H, Dv), dtype=torch.float32, device=dev)
    _check(o, "o", torch.float32, (B, T, H, Dv), dev)
    if S_T is None:
        S_T = torch.empty((B, H, Dv, Dk), dtype=torch.float32, device=dev)
    _check(S_T, "S_T", torch.float32, (B, H, Dv, Dk), dev)
    if status is not None:
        _check(status, "status", torch.int32, (1,), dev)
    rc = _lib.gdn_prefill_static_ws(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0),
                                    _ptr(o), _ptr(S_T), B, T, H, Dk, Dv, int(chunk), _ptr(status),
                                    _stream_handle(dev))
    if rc != GDN_OK:
        raise GDNError(rc, "gdn_prefill_static_ws")
    return o, S_T


def decode_step(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor,
                beta: torch.Tensor, S: torch.Tensor, *, o: Optional[torch.Tensor] = None,
                status: Optional[torch.Tensor] = None, qk_l2norm: bool = False,
                q_scale: float = 1.0, o_bf16: bool = False) -> torch.Tensor:
    """One decode step; S [B,H,Dv,Dk] fp32 is updated in place.  Returns o [B,H,Dv]
    (fp32, or bf16 with ``o_bf16``).

    q, k [B,H,Dk] bf16; v [B,H,Dv] bf16; g, beta [B,H] fp32.  The fused options
    (``qk_l2norm``, ``q_scale``, ``o_bf16``; gdn_decode_ex) need Dk = Dv = 128
    or 64."""
    if q.dim() != 3:
        raise ValueError("q must be [B,H,Dk]")
    B, H, Dk = q.shape
    Dv = v.shape[-1]
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("gdn.decode_step runs on CUDA tensors only (no CPU path)")
    _check(q, "q", torch.bfloat16, (B, H, Dk), dev)
    _check(k, "k", torch.bfloat16, (B, H, Dk), dev)
    _check(v, "v", torch.bfloat16, (B, H, Dv), dev)
    _check(g, "g", torch.float32, (B, H), dev)
    _check(beta, "beta", torch.float32, (B, H), dev)
    _check(S, "S", torch.float32, (B, H, Dv, Dk), dev)
    o_dtype = torch.bfloat16 if o_bf16 else torch.float32
    if o is None:
        o = torch.empty((B, H, Dv), dtype=o_dtype, device=dev)
    _check(o, "o", o_dtype, (B, H, Dv), dev)
    opts = _options(qk_l2norm, q_scale, o_bf16)
    if opts is None:
        rc = _lib.gdn_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S), _ptr(o),
                                  B, H, Dk, Dv, _ptr(status), _stream_handle(dev))
    else:
        rc = _lib.gdn_decode_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S), _ptr(o),
                                B, 1, H, Dk, Dv, opts, _ptr(status), _stream_handle(dev))
    if rc != GDN_OK:
        raise GDNError(rc, "gdn_decode_step")
    return o


def decode_tokens(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor,
                  beta: torch.Tensor, S: torch.Tensor, *, o: Optional[torch.Tensor] = None,
                  status: Optional[torch.Tensor] = None, qk_l2norm: bool = False,
                  q_scale: float = 1.0, o_bf16: bool = False) -> torch.Tensor:
    """T decode tokens per sequence in one call; S [B,H,Dv,Dk] fp32 is updated in
    place (read and written once).  Returns o [B,T,H,Dv] (fp32, or bf16 with
    ``o_bf16``).

    q, k [B,T,H,Dk] bf16; v [B,T,H,Dv] bf16; g, beta [B,T,H] fp32.  The fused
    options need Dk = Dv = 128 or 64."""
    if q.dim() != 4:
        raise ValueError("q must be [B,T,H,Dk]")
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("gdn.decode_tokens runs on CUDA tensors only (no CPU path)")
    _check(q, "q", torch.bfloat16, (B, T, H, Dk), dev)
    _check(k, "k", torch.bfloat16, (B, T, H, Dk), dev)
    _check(v, "v", torch.bfloat16, (B, T, H, Dv), dev)
    _check(g, "g", torch.float32, (B, T, H), dev)
    _check(beta, "beta", torch.float32, (B, T, H), dev)
    _check(S, "S", torch.float32, (B, H, Dv, Dk), dev)
    o_dtype = torch.bfloat16 if o_bf16 else torch.float32
    if o is None:
        o = torch.empty((B, T, H, Dv), dtype=o_dtype, device=dev)
    _check(o, "o", o_dtype, (B, T, H, Dv), dev)
    opts = _options(qk_l2norm, q_scale, o_bf16)
    if opts is None:
        rc = _lib.gdn_decode_tokens(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S),
                                    _ptr(o), B, T, H, Dk, Dv, _ptr(status), _stream_handle(dev))
    else:
        rc = _lib.gdn_decode_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S), _ptr(o),
                                B, T, H, Dk, Dv, opts, _ptr(status), _stream_handle(dev))
    if rc != GDN_OK:
        raise GDNError(rc, "gdn_decode_tokens")
    return o


def query_status(status: torch.Tensor) -> int:
    """Synchronises the current stream and returns the device status word."""
    return int(_lib.gdn_query_status(_ptr(status), _stream_handle(status.device)))


def kda_prefill(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor,
                beta: torch.Tensor, S0: Optional[torch.Tensor] = None, *,
                o: Optional[torch.Tensor] = None, S_T: Optional[torch.Tensor] = None,
                status: Optional[torch.Tensor] = None, qk_l2norm: bool = False,
                q_scale: float = 1.0, o_bf16: bool = False) -> Tuple[torch.Tensor, torch.Tensor]:
    """Per-channel-gate (KDA) prefill: returns (o [B,T,H,Dv] fp32, or bf16 with
    ``o_bf16``, S_T [B,H,Dv,Dk] fp32).

    q, k [B,T,H,Dk] bf16; v [B,T,H,Dv] bf16; g [B,T,H,Dk] fp32 (log decay per key
    channel); beta [B,T,H] fp32; S0 [B,H,Dv,Dk] fp32 or None (zeros).  ``S_T``
    may be ``S0`` (in place).  ``qk_l2norm`` / ``q_scale`` normalise q and k per
    token and head and scale q inside the kernel, and ``o_bf16`` writes o as bf16
    (gdn_kda_prefill_ex; Dk = 128).  Dk = 128 runs the chunked tensor-core kernel
    (Dv 64, 128 or 256); Dk = 64 or 256 the row kernel.  Launches on the current
    stream."""
    if q.dim() != 4:
        raise ValueError("q must be [B,T,H,Dk]")
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("gdn.kda_prefill runs on CUDA tensors only (no CPU path)")
    _check(q, "q", torch.bfloat16, (B, T, H, Dk), dev)
    _check(k, "k", torch.bfloat16, (B, T, H, Dk), dev)
    _check(v, "v", torch.bfloat16, (B, T, H, Dv), dev)
    _check(g, "g", torch.float32, (B, T, H, Dk), dev)
    _check(beta, "beta", torch.float32, (B, T, H), dev)
    if S0 is not None:
        _check(S0, "S0", torch.float32, (B, H, Dv, Dk), dev)
    o_dtype = torch.bfloat16 if o_bf16 else torch.float32
    if o is None:
        o = torch.empty((B, T, H, Dv), dtype=o_dtype, device=dev)
    _check(o, "o", o_dtype, (B, T, H, Dv), dev)
    if S_T is None:
        S_T = torch.empty((B, H, Dv, Dk), dtype=torch.float32, device=dev)
    _check(S_T, "S_T", torch.float32, (B, H, Dv, Dk), dev)
    opts = _options(qk_l2norm, q_scale, o_bf16)
    if opts is None:
        rc = _lib.gdn_kda_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0), _ptr(o),
                                  _ptr(S_T), B, T, H, Dk, Dv, _ptr(status), _stream_handle(dev))
    else:
        rc = _lib.gdn_kda_prefill_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0), _ptr(o),
                                     _ptr(S_T), B, T, H, Dk, Dv, opts, _ptr(status), _stream_handle(dev))
    if rc != GDN_OK:
        raise GDNError(rc, "gdn_kda_prefill")
    return o, S_T


def kda_prefill_varlen(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor,
                       beta: torch.Tensor, cu_seqlens: torch.Tensor,
                       S0: Optional[torch.Tensor] = None, *, o: Optional[torch.Tensor] = None,
                       S_T: Optional[torch.Tensor] = None,
                       status: Optional[torch.Tensor] = None, snap_every: int = 0,
                       snaps: Optional[torch.Tensor] = None, qk_l2norm: bool = False,
                       q_scale: float = 1.0, o_bf16: bool = False):
    """Per-channel-gate prefill of N packed sequences (gdn_kda_prefill_varlen):
    q, k [total_T,H,128] bf16; v [total_T,H,Dv] bf16 (Dv 64, 128 or 256);
    g [total_T,H,128] fp32; beta [total_T,H] fp32; cu_seqlens int32 [N+1] on
    the device.  Returns (o [total_T,H,Dv] fp32 or bf16, S_T [N,H,Dv,128] fp32), and
    with ``snap_every`` (a multiple of 32) the state snapshots as in
    ``prefill_varlen``.  ``qk_l2norm``, ``q_scale`` and ``o_bf16`` as in
    ``kda_prefill``."""
    if q.dim() != 3:
        raise ValueError("q must be [total_T,H,Dk]")
    total_T, H, Dk = q.shape
    Dv = v.shape[-1]
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("gdn.kda_prefill_varlen runs on CUDA tensors only (no CPU path)")
    if cu_seqlens.dim() != 1 or cu_seqlens.numel() < 1:
        raise ValueError("cu_seqlens must be [N+1]")
    N = cu_seqlens.numel() - 1
    _check(cu_seqlens, "cu_seqlens", torch.int32, (N + 1,), dev)
    _check(q, "q", torch.bfloat16, (total_T, H, Dk), dev)
    _check(k, "k", torch.bfloat16, (total_T, H, Dk), dev)
    _check(v, "v", torch.bfloat16, (total_T, H, Dv), dev)
    _check(g, "g", torch.float32, (total_T, H, Dk), dev)
    _check(beta, "beta", torch.float32, (total_T, H), dev)
    if S0 is not None:
        _check(S0, "S0", torch.float32, (N, H, Dv, Dk), dev)
    o_dtype = torch.bfloat16 if o_bf16 else torch.float32
    if o is None:
        o = torch.empty((total_T, H, Dv), dtype=o_dtype, device=dev)
    _check(o, "o", o_dtype, (total_T, H, Dv), dev)
    if S_T is None:
        S_T = torch.empty((N, H, Dv, Dk), dtype=torch.float32, device=dev)
    _check(S_T, "S_T", torch.float32, (N, H, Dv, Dk), dev)
    if status is not None:
        _check(status, "status", torch.int32, (1,), dev)
    n_snaps = 0
    if snap_every:
        if snaps is None:
            lens = (cu_seqlens[1:] - cu_seqlens[:-1]).cpu()
            n_snaps = int((lens // int(snap_every)).sum())
            snaps = torch.empty((n_snaps, H, Dv, Dk), dtype=torch.float32, device=dev)
        n_snaps = snaps.shape[0]
        _check(snaps, "snaps", torch.float32, (n_snaps, H, Dv, Dk), dev)
    else:
        snaps = None
    opts = _options(qk_l2norm, q_scale, o_bf16)
    if opts is None:
        rc = _lib.gdn_kda_prefill_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0),
                                         _ptr(o), _ptr(S_T), _ptr(cu_seqlens), N, total_T, H, Dk,
                                         Dv, _ptr(snaps), int(snap_every), n_snaps, _ptr(status),
                                         _stream_handle(dev))
    else:
        rc = _lib.gdn_kda_prefill_varlen_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                            _ptr(S0), _ptr(o), _ptr(S_T), _ptr(cu_seqlens), N,
                                            total_T, H, Dk, Dv, _ptr(snaps), int(snap_every),
                                            n_snaps, opts, _ptr(status), _stream_handle(dev))
    if rc != GDN_OK:
        raise GDNError(rc, "gdn_kda_prefill_varlen")
    return (o, S_T) if snaps is None else (o, S_T, snaps)


def kda_decode(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor,
               beta: torch.Tensor, S: torch.Tensor, *, o: Optional[torch.Tensor] = None,
               status: Optional[torch.Tensor] = None, qk_l2norm: bool = False,
               q_scale: float = 1.0, o_bf16: bool = False) -> torch.Tensor:
    """Per-channel-gate (KDA) decode; S [B,H,Dv,Dk] fp32 is updated in place.

    One token: q, k [B,H,Dk], v [B,H,Dv], g [B,H,Dk], beta [B,H] -> o [B,H,Dv].
    T tokens: the same with a T axis after B ([B,T,H,...]) -> o [B,T,H,Dv].
    ``qk_l2norm`` / ``q_scale`` / ``o_bf16`` as for ``kda_prefill``
    (gdn_kda_decode_ex; 128 x 128 or 64 x 64)."""
    one = q.dim() == 3
    if one:
        q, k, v, g, beta = (x.unsqueeze(1) for x in (q, k, v, g, beta))
        if o is not None:
            o = o.unsqueeze(1)
    if q.dim() != 4:
        raise ValueError("q must be [B,H,Dk] or [B,T,H,Dk]")
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("gdn.kda_decode runs on CUDA tensors only (no CPU path)")
    _check(q, "q", torch.bfloat16, (B, T, H, Dk), dev)
    _check(k, "k", torch.bfloat16, (B, T, H, Dk), dev)
    _check(v, "v", torch.bfloat16, (B, T, H, Dv), dev)
    _check(g, "g", torch.float32, (B, T, H, Dk), dev)
    _check(beta, "beta", torch.float32, (B, T, H), dev)
    _check(S, "S", torch.float32, (B, H, Dv, Dk), dev)
    o_dtype = torch.bfloat16 if o_bf16 else torch.float32
    if o is None:
        o = torch.empty((B, T, H, Dv), dtype=o_dtype, device=dev)
    _check(o, "o", o_dtype, (B, T, H, Dv), dev)
    opts = _options(qk_l2norm, q_scale, o_bf16)
    if opts is None:
        rc = _lib.gdn_kda_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S), _ptr(o),
                                 B, T, H, Dk, Dv, _ptr(status), _stream_handle(dev))
    else:
        rc = _lib.gdn_kda_decode_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S), _ptr(o),
                                    B, T, H, Dk, Dv, opts, _ptr(status), _stream_handle(dev))
    if rc != GDN_OK:
        raise GDNError(rc, "gdn_kda_decode")
    return o[:, 0] if one else o


def raw_prefill(*args) -> int:
    """Direct call of the C entry point with raw integers/pointers (tests use it
    to exercise argument validation without any tensor)."""
    return int(_lib.gdn_prefill(*args))


def raw_prefill_ex(*args) -> int:
    return int(_lib.gdn_prefill_ex(*args))


def raw_decode_ex(*args) -> int:
    return int(_lib.gdn_decode_ex(*args))


def raw_prefill_varlen(*args) -> int:
    return int(_lib.gdn_prefill_varlen(*args))


def raw_prefill_static_ws(*args) -> int:
    return int(_lib.gdn_prefill_static_ws(*args))


def raw_prefill_ws(*args) -> int:
    return int(_lib.gdn_prefill_ws(*args))


def raw_decode_tokens(*args) -> int:
    return int(_lib.gdn_decode_tokens(*args))


def raw_decode_step(*args) -> int:
    return int(_lib.gdn_decode_step(*args))


def raw_kda_prefill(*args) -> int:
    return int(_lib.gdn_kda_prefill(*args))


def raw_kda_decode(*args) -> int:
    return int(_lib.gdn_kda_decode(*args))


def raw_kda_prefill_ex(*args) -> int:
    return int(_lib.gdn_kda_prefill_ex(*args))


def raw_kda_decode_ex(*args) -> int:
    return int(_lib.gdn_kda_decode_ex(*args))


def raw_kda_prefill_varlen(*args) -> int:
    return int(_lib.gdn_kda_prefill_varlen(*args))


def raw_prefill_varlen_ex(*args) -> int:
    return int(_lib.gdn_prefill_varlen_ex(*args))


def raw_kda_prefill_varlen_ex(*args) -> int:
    return int(_lib.gdn_kda_prefill_varlen_ex(*args))
