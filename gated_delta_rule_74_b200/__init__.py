"""gated_delta_rule_74_b200: B200 (sm_100a) Kimi Delta Attention (KDA).

Thin ctypes binding over libkda.so, whose C ABI is declared in include/kda.h.
The functions here only marshal torch CUDA tensors into pointers and sizes and
call the library on the current torch stream; every step of the computation runs
in the library's CUDA kernels.  There is no fallback: if libkda.so is missing or a
call fails, an exception is raised.

    out, hT = kda_chunk_fwd(q, k, v, g, beta, h0=None, cu_seqlens=None)
    out     = kda_decode_step(q, k, v, g, beta, S)        # S updated in place
    grads   = kda_chunk_bwd(q, k, v, g, beta, dout, h0=None, dhT=None, cu_seqlens=None)
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

import torch

__all__ = ["kda_chunk_fwd", "kda_chunk_fwd_fused", "kda_chunk_bwd", "kda_device_status",
           "kda_decode_chunk", "kda_decode_step", "kda_decode_tokens", "kda_status_string", "kda_version",
           "kda_launch_count",
           "lib", "library_path", "header_symbols", "KdaError",
           "KDA_OK", "KDA_ERR_INVALID_ARG", "KDA_ERR_UNSUPPORTED", "KDA_ERR_CUDA",
           "KDA_ERR_TIMEOUT", "KDA_BF16", "KDA_F32", "KDA_OP_CHUNK_FWD", "KDA_OP_CHUNK_BWD",
           "kda_workspace_size", "kda_pool_usage"]

_PKG = os.path.dirname(os.path.abspath(__file__))
_ROOT = os.path.dirname(_PKG)
_SO = os.path.join(_PKG, "libkda.so")
_HEADER = os.path.join(_ROOT, "include", "kda.h")

KDA_OK, KDA_ERR_INVALID_ARG, KDA_ERR_UNSUPPORTED, KDA_ERR_CUDA, KDA_ERR_TIMEOUT = 0, -1, -2, -3, -4
KDA_BF16, KDA_F32 = 0, 1
KDA_OP_CHUNK_FWD, KDA_OP_CHUNK_BWD = 0, 1

_DTYPES = {torch.bfloat16: KDA_BF16, torch.float32: KDA_F32}
_lib = None


class KdaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {kda_status_string(status)} ({status})")


def _check_status(rc: int, fn: str = "kda_timing") -> None:
    if rc != 0:
        raise KdaError(fn, rc)


def library_path() -> str:
    return _SO


def lib() -> ctypes.CDLL:
    """Load libkda.so (built in-tree by gated_delta_rule_74_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_SO):
            raise RuntimeError(f"libkda.so is not built ({_SO}); run "
                               "`python -m gated_delta_rule_74_b200.build`")
        L = ctypes.CDLL(_SO)
        vp, fp, ip = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int
        L.kda_chunk_fwd.argtypes = [vp, vp, vp, fp, fp, fp, vp, vp, fp,
                                    ip, ip, ip, ip, ip, ip, vp]
        L.kda_chunk_fwd.restype = ctypes.c_int
        L.kda_chunk_fwd_noalloc.argtypes = [vp, vp, vp, fp, fp, fp, vp, vp, fp,
                                            ip, ip, ip, ip, ip, ip, vp]
        L.kda_chunk_fwd_noalloc.restype = ctypes.c_int
        L.kda_decode_step.argtypes = [vp, vp, vp, fp, fp, fp, vp, ip, ip, ip, ip, ip, vp]
        L.kda_decode_step.restype = ctypes.c_int
        L.kda_decode_tokens.argtypes = [vp, vp, vp, fp, fp, fp, vp, ip, ip, ip, ip, ip, ip, vp]
        L.kda_decode_tokens.restype = ctypes.c_int
        L.kda_decode_chunk.argtypes = [vp, vp, vp, fp, fp, fp, vp, ip, ip, ip, ip, ip, ip, vp]
        L.kda_decode_chunk.restype = ctypes.c_int
        L.kda_decode_tokens_grouped.argtypes = [vp, vp, vp, fp, fp, fp, vp] + [ip] * 7 + [vp]
        L.kda_decode_tokens_grouped.restype = ctypes.c_int
        L.kda_chunk_fwd_grouped.argtypes = [vp, vp, vp, fp, fp, fp, vp, vp, fp] + [ip] * 7 + [vp]
        L.kda_chunk_fwd_grouped.restype = ctypes.c_int
        L.kda_chunk_fwd_fused.argtypes = [vp, vp, vp, fp, fp, ip, fp, fp, vp, fp, vp, vp, fp] + \
            [ip] * 6 + [vp]
        L.kda_chunk_fwd_fused.restype = ctypes.c_int
        L.kda_chunk_bwd.argtypes = [vp, vp, vp, fp, fp, fp, vp, vp, fp,
                                    fp, fp, fp, fp, fp, fp] + [ip] * 6 + [vp]
        L.kda_chunk_bwd.restype = ctypes.c_int
        L.kda_chunk_bwd_grouped.argtypes = [vp, vp, vp, fp, fp, fp, vp, vp, fp,
                                            fp, fp, fp, fp, fp, fp] + [ip] * 7 + [vp]
        L.kda_chunk_bwd_grouped.restype = ctypes.c_int
        L.kda_chunk_bwd_recurrent.argtypes = L.kda_chunk_bwd_grouped.argtypes
        L.kda_chunk_bwd_recurrent.restype = ctypes.c_int
        L.kda_device_status.argtypes = [ip]
        L.kda_device_status.restype = ctypes.c_int
        L.kda_selftest_bounded_wait.argtypes = [ctypes.c_uint, vp]
        L.kda_selftest_bounded_wait.restype = ctypes.c_int
        L.kda_status_string.argtypes = [ctypes.c_int]
        L.kda_status_string.restype = ctypes.c_char_p
        L.kda_version.argtypes = []
        L.kda_version.restype = ctypes.c_int
        L.kda_launch_count.argtypes = []
        L.kda_launch_count.restype = ctypes.c_ulonglong
        L.kda_prefill_plan.argtypes = [ctypes.c_int] * 5 + [ctypes.POINTER(ctypes.c_int)] * 2
        L.kda_prefill_plan.restype = ctypes.c_int
        L.kda_timing_start.argtypes = []
        L.kda_timing_start.restype = ctypes.c_int
        L.kda_timing_stop.argtypes = []
        L.kda_timing_stop.restype = ctypes.c_int
        L.kda_timing_read.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_ulonglong),
                                      ctypes.POINTER(ctypes.c_double)]
        L.kda_timing_read.restype = ctypes.c_int
        sz = ctypes.c_size_t
        L.kda_workspace_size.argtypes = [ctypes.c_int] * 9 + [ctypes.POINTER(sz)]
        L.kda_workspace_size.restype = ctypes.c_int
        L.kda_chunk_fwd_ws.argtypes = [vp, vp, vp, fp, fp, fp, vp, vp, fp] + [ip] * 7 + [vp, sz, vp]
        L.kda_chunk_fwd_ws.restype = ctypes.c_int
        L.kda_chunk_bwd_ws.argtypes = [vp, vp, vp, fp, fp, fp, vp, vp, fp,
                                       fp, fp, fp, fp, fp, fp] + [ip] * 7 + [vp, sz, vp]
        L.kda_chunk_bwd_ws.restype = ctypes.c_int
        L.kda_pool_usage.argtypes = [ip, ctypes.POINTER(ctypes.c_ulonglong)]
        L.kda_pool_usage.restype = ctypes.c_int
        _lib = L
    return _lib


def header_symbols() -> list[str]:
    """Names of the functions include/kda.h declares."""
    with open(_HEADER) as f:
        text = f.read()
    return re.findall(r"^KDA_API\s+[\w\s\*]*?\b(kda_\w+)\s*\(", text, flags=re.M)


def kda_workspace_size(op: int, B: int, T: int, H: int, dk: int, dv: int, packed: bool = False,
                       dtype: int = KDA_BF16, sms: int = 0) -> int:
    """Workspace bytes of one kda_chunk_fwd_ws (op KDA_OP_CHUNK_FWD) or kda_chunk_bwd_ws
    (KDA_OP_CHUNK_BWD) call; sms = 0 asks the current device."""
    out = ctypes.c_size_t(0)
    rc = lib().kda_workspace_size(int(op), int(B), int(T), int(H), int(dk), int(dv),
                                  1 if packed else 0, int(dtype), int(sms), ctypes.byref(out))
    if rc != KDA_OK:
        raise KdaError("kda_workspace_size", rc)
    return int(out.value)


def kda_pool_usage(reset: bool = False) -> int:
    """Most bytes the library pool of the current device has had in use at once."""
    out = ctypes.c_ulonglong(0)
    rc = lib().kda_pool_usage(1 if reset else 0, ctypes.byref(out))
    if rc != KDA_OK:
        raise KdaError("kda_pool_usage", rc)
    return int(out.value)


def _workspace_args(workspace: Optional[torch.Tensor]):
    if workspace is None:
        return None, 0
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    return _ptr(workspace), workspace.numel() * workspace.element_size()


def kda_status_string(status: int) -> str:
    return lib().kda_status_string(int(status)).decode()


def kda_version() -> int:
    return int(lib().kda_version())


def kda_device_status(reset: bool = True) -> int:
    """KDA_OK, or KDA_ERR_TIMEOUT if a bounded device-side wait of the library's kernels
    gave up since the last reset (synchronizes the device; see include/kda.h)."""
    rc = int(lib().kda_device_status(1 if reset else 0))
    if rc not in (KDA_OK, KDA_ERR_TIMEOUT):
        raise KdaError("kda_device_status", rc)
    return rc


def kda_selftest_bounded_wait(polls: int = 1000, stream=None) -> None:
    """Launch the self-test whose wait nothing completes (see include/kda.h)."""
    rc = lib().kda_selftest_bounded_wait(int(polls), _stream(stream))
    if rc != KDA_OK:
        raise KdaError("kda_selftest_bounded_wait", rc)


def kda_launch_count() -> int:
    """Kernels launched by libkda in this process so far."""
    return int(lib().kda_launch_count())


def kda_prefill_plan(B: int, T: int, H: int, packed: bool = False, sms: int = 148) -> tuple:
    """(chunks per segment, chunks of a half point) that kda_chunk_fwd's split takes for
    B sequences of T tokens (packed: T tokens in B documents) over H heads on `sms` SMs;
    (0, 0) when sequences are not split.  Host only."""
    G, half = ctypes.c_int(0), ctypes.c_int(0)
    rc = lib().kda_prefill_plan(B, T, H, int(bool(packed)), sms, ctypes.byref(G),
                                ctypes.byref(half))
    _check_status(rc, "kda_prefill_plan")
    return int(G.value), int(half.value)


KERNEL_KINDS = {"prep": 0, "state": 1, "combine": 2, "fused": 3, "simt": 4, "decode": 5,
                "bwd": 6, "bwd_prep": 7, "bwd_chain": 8, "bwd_grad": 9}


def kda_timing_start() -> None:
    """Start bracketing every library kernel launch with CUDA events."""
    _check_status(lib().kda_timing_start())


def kda_timing_stop() -> None:
    _check_status(lib().kda_timing_stop())


def kda_timing_read() -> dict:
    """{kind: (launches, total_ms)} since kda_timing_start(); waits for the events."""
    res = {}
    for name, kind in KERNEL_KINDS.items():
        n = ctypes.c_ulonglong(0)
        ms = ctypes.c_double(0.0)
        _check_status(lib().kda_timing_read(kind, ctypes.byref(n), ctypes.byref(ms)))
        res[name] = (int(n.value), float(ms.value))
    return res


def _decay_group(g: torch.Tensor, dk: int) -> int:
    """Channels per decay value implied by g's last dimension."""
    n = g.shape[-1]
    if n < 1 or dk % n != 0 or (dk // n) & (dk // n - 1):
        raise ValueError(f"g's last dimension {n} must be dk / G with G a power of two")
    return dk // n


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(name: str, t: torch.Tensor, dtype=None, shape=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def kda_chunk_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor,
                  beta: torch.Tensor, h0: Optional[torch.Tensor] = None,
                  cu_seqlens: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                  hT: Optional[torch.Tensor] = None, output_final_state: bool = True,
                  stream=None, noalloc: bool = False, workspace: Optional[torch.Tensor] = None):
    """KDA prefill (chunked form).  q, k [B,T,H,dk]; v [B,T,H,dv]; g [B,T,H,dk] f32
    (or [B,T,H,dk/G] for one decay per group of G key channels, G a power of two:
    kda_chunk_fwd_grouped); beta [B,T,H] f32; h0 [Nseq,H,dk,dv] f32 or None;
    cu_seqlens int32 [Nseq+1] on the device, or None.  Returns (out, hT) (hT None
    if output_final_state is False and no hT buffer was given).  noalloc=True calls
    kda_chunk_fwd_noalloc instead (per-channel decay only); a ``workspace`` tensor
    (kda_workspace_size bytes, e.g. torch.uint8) calls kda_chunk_fwd_ws on it."""
    if q.dim() != 4:
        raise ValueError("q must be [B, T, H, dk]")
    Bt, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = _DTYPES.get(q.dtype)
    if dt is None:
        raise ValueError(f"unsupported dtype {q.dtype}")
    _check("q", q)
    _check("k", k, q.dtype, (Bt, T, H, dk))
    _check("v", v, q.dtype, (Bt, T, H, dv))
    G = _decay_group(g, dk)
    _check("g", g, torch.float32, (Bt, T, H, dk // G))
    _check("beta", beta, torch.float32, (Bt, T, H))
    if cu_seqlens is not None:
        _check("cu_seqlens", cu_seqlens, torch.int32)
        if Bt != 1:
            raise ValueError("packed inputs (cu_seqlens) must have B == 1")
        nseq = cu_seqlens.numel() - 1
    else:
        nseq = Bt
    if h0 is not None:
        _check("h0", h0, torch.float32, (nseq, H, dk, dv))
    if out is None:
        out = torch.empty((Bt, T, H, dv), dtype=q.dtype, device=q.device)
    _check("out", out, q.dtype, (Bt, T, H, dv))
    if hT is None and output_final_state:
        hT = torch.empty((nseq, H, dk, dv), dtype=torch.float32, device=q.device)
    if hT is not None:
        _check("hT", hT, torch.float32, (nseq, H, dk, dv))
    if noalloc and G != 1:
        raise ValueError("kda_chunk_fwd_noalloc takes one decay per key channel")
    if workspace is not None:
        wp, wb = _workspace_args(workspace)
        rc = lib().kda_chunk_fwd_ws(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0),
                                    _ptr(cu_seqlens), _ptr(out), _ptr(hT), nseq, T, H, dk, dv, G,
                                    dt, wp, wb, _stream(stream))
        if rc != KDA_OK:
            raise KdaError("kda_chunk_fwd_ws", rc)
        return out, hT
    if G == 1:
        fn = lib().kda_chunk_fwd_noalloc if noalloc else lib().kda_chunk_fwd
        rc = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0),
                _ptr(cu_seqlens), _ptr(out), _ptr(hT), nseq, T, H, dk, dv, dt, _stream(stream))
    else:
        rc = lib().kda_chunk_fwd_grouped(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                         _ptr(h0), _ptr(cu_seqlens), _ptr(out), _ptr(hT),
                                         nseq, T, H, dk, dv, G, dt, _stream(stream))
    if rc != KDA_OK:
        raise KdaError("kda_chunk_fwd_noalloc" if noalloc else "kda_chunk_fwd", rc)
    return out, hT


def kda_chunk_fwd_fused(q_raw: torch.Tensor, k_raw: torch.Tensor, v: torch.Tensor,
                        g: torch.Tensor, beta: torch.Tensor,
                        conv_q: Optional[torch.Tensor] = None,
                        conv_k: Optional[torch.Tensor] = None,
                        gate: Optional[torch.Tensor] = None, h0: Optional[torch.Tensor] = None,
                        cu_seqlens: Optional[torch.Tensor] = None,
                        out: Optional[torch.Tensor] = None, hT: Optional[torch.Tensor] = None,
                        output_final_state: bool = True, stream=None):
    """KDA prefill with the q/k prep and the output gate fused (bf16 only):
    q = dk^-1/2 n(conv_q * q_raw), k = n(conv_k * k_raw) (causal per-channel convolutions
    of width W, conv_* [H, dk, W] f32, n = L2 normalisation per token and head),
    out = o * sigmoid(gate) (gate [B,T,H,dv] bf16 or None).  Returns (out, hT)."""
    if q_raw.dim() != 4:
        raise ValueError("q_raw must be [B, T, H, dk]")
    Bt, T, H, dk = q_raw.shape
    dv = v.shape[-1]
    dt = _DTYPES.get(q_raw.dtype)
    if dt is None:
        raise ValueError(f"unsupported dtype {q_raw.dtype}")
    _check("q_raw", q_raw)
    _check("k_raw", k_raw, q_raw.dtype, (Bt, T, H, dk))
    _check("v", v, q_raw.dtype, (Bt, T, H, dv))
    _check("g", g, torch.float32, (Bt, T, H, dk))
    _check("beta", beta, torch.float32, (Bt, T, H))
    W = 0
    if (conv_q is None) != (conv_k is None):
        raise ValueError("give both conv_q and conv_k, or neither")
    if conv_q is not None:
        W = conv_q.shape[-1]
        _check("conv_q", conv_q, torch.float32, (H, dk, W))
        _check("conv_k", conv_k, torch.float32, (H, dk, W))
    if gate is not None:
        _check("gate", gate, q_raw.dtype, (Bt, T, H, dv))
    if cu_seqlens is not None:
        _check("cu_seqlens", cu_seqlens, torch.int32)
        if Bt != 1:
            raise ValueError("packed inputs (cu_seqlens) must have B == 1")
        nseq = cu_seqlens.numel() - 1
    else:
        nseq = Bt
    if h0 is not None:
        _check("h0", h0, torch.float32, (nseq, H, dk, dv))
    if out is None:
        out = torch.empty((Bt, T, H, dv), dtype=q_raw.dtype, device=q_raw.device)
    _check("out", out, q_raw.dtype, (Bt, T, H, dv))
    if hT is None and output_final_state:
        hT = torch.empty((nseq, H, dk, dv), dtype=torch.float32, device=q_raw.device)
    if hT is not None:
        _check("hT", hT, torch.float32, (nseq, H, dk, dv))
    rc = lib().kda_chunk_fwd_fused(_ptr(q_raw), _ptr(k_raw), _ptr(v), _ptr(conv_q), _ptr(conv_k),
                                   W, _ptr(g), _ptr(beta), _ptr(gate), _ptr(h0),
                                   _ptr(cu_seqlens), _ptr(out), _ptr(hT), nseq, T, H, dk, dv, dt,
                                   _stream(stream))
    if rc != KDA_OK:
        raise KdaError("kda_chunk_fwd_fused", rc)
    return out, hT


def kda_chunk_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor,
                  beta: torch.Tensor, dout: torch.Tensor, h0: Optional[torch.Tensor] = None,
                  dhT: Optional[torch.Tensor] = None, cu_seqlens: Optional[torch.Tensor] = None,
                  grads: Optional[dict] = None, stream=None,
                  workspace: Optional[torch.Tensor] = None, recurrent: bool = False) -> dict:
    """Gradients of L = sum(out * dout) + sum(hT * dhT) for kda_chunk_fwd with the same
    inputs.  g [B,T,H,dk] f32, or [B,T,H,dk/G] for one decay per group of G key channels
    (kda_chunk_bwd_grouped; dg then has g's shape).  dout has out's shape and dtype; dhT
    [Nseq,H,dk,dv] f32 or None.  Returns a dict of fp32 tensors dq, dk, dv, dg, dbeta, dh0
    (dh0 None when h0 is None); ``grads`` may hold preallocated outputs under those names;
    a ``workspace`` tensor (kda_workspace_size bytes) calls kda_chunk_bwd_ws on it;
    ``recurrent`` calls kda_chunk_bwd_recurrent (the fp32 reverse sweep) instead."""
    if q.dim() != 4:
        raise ValueError("q must be [B, T, H, dk]")
    Bt, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = _DTYPES.get(q.dtype)
    if dt is None:
        raise ValueError(f"unsupported dtype {q.dtype}")
    _check("q", q)
    _check("k", k, q.dtype, (Bt, T, H, dk))
    _check("v", v, q.dtype, (Bt, T, H, dv))
    G = _decay_group(g, dk)
    _check("g", g, torch.float32, (Bt, T, H, dk // G))
    _check("beta", beta, torch.float32, (Bt, T, H))
    _check("dout", dout, q.dtype, (Bt, T, H, dv))
    if cu_seqlens is not None:
        _check("cu_seqlens", cu_seqlens, torch.int32)
        if Bt != 1:
            raise ValueError("packed inputs (cu_seqlens) must have B == 1")
        nseq = cu_seqlens.numel() - 1
    else:
        nseq = Bt
    if h0 is not None:
        _check("h0", h0, torch.float32, (nseq, H, dk, dv))
    if dhT is not None:
        _check("dhT", dhT, torch.float32, (nseq, H, dk, dv))
    shapes = {"dq": (Bt, T, H, dk), "dk": (Bt, T, H, dk), "dv": (Bt, T, H, dv),
              "dg": (Bt, T, H, dk // G), "dbeta": (Bt, T, H), "dh0": (nseq, H, dk, dv)}
    res = dict(grads or {})
    for name, shp in shapes.items():
        if name == "dh0" and h0 is None and res.get(name) is None:
            res[name] = None
            continue
        if res.get(name) is None:
            res[name] = torch.empty(shp, dtype=torch.float32, device=q.device)
        _check(name, res[name], torch.float32, shp)
    args = [_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0), _ptr(cu_seqlens),
            _ptr(dout), _ptr(dhT), _ptr(res["dq"]), _ptr(res["dk"]), _ptr(res["dv"]),
            _ptr(res["dg"]), _ptr(res["dbeta"]), _ptr(res["dh0"]), nseq, T, H, dk, dv]
    if recurrent:
        if workspace is not None:
            raise ValueError("the recurrent backward takes no workspace")
        rc = lib().kda_chunk_bwd_recurrent(*args, G, dt, _stream(stream))
        if rc != KDA_OK:
            raise KdaError("kda_chunk_bwd_recurrent", rc)
        return res
    if workspace is not None:
        wp, wb = _workspace_args(workspace)
        rc = lib().kda_chunk_bwd_ws(*args, G, dt, wp, wb, _stream(stream))
        if rc != KDA_OK:
            raise KdaError("kda_chunk_bwd_ws", rc)
        return res
    if G == 1:
        rc = lib().kda_chunk_bwd(*args, dt, _stream(stream))
    else:
        rc = lib().kda_chunk_bwd_grouped(*args, G, dt, _stream(stream))
    if rc != KDA_OK:
        raise KdaError("kda_chunk_bwd", rc)
    return res


def kda_decode_step(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor,
                    beta: torch.Tensor, S: torch.Tensor, out: Optional[torch.Tensor] = None,
                    stream=None) -> torch.Tensor:
    """One KDA decode step.  q, k [N,H,dk]; v [N,H,dv]; g [N,H,dk] f32; beta [N,H] f32;
    S [N,H,dk,dv] f32, updated in place.  Returns out [N,H,dv]."""
    if q.dim() != 3:
        raise ValueError("q must be [N, H, dk]")
    N, H, dk = q.shape
    dv = v.shape[-1]
    dt = _DTYPES.get(q.dtype)
    if dt is None:
        raise ValueError(f"unsupported dtype {q.dtype}")
    _check("q", q)
    _check("k", k, q.dtype, (N, H, dk))
    _check("v", v, q.dtype, (N, H, dv))
    _check("g", g, torch.float32, (N, H, dk))
    _check("beta", beta, torch.float32, (N, H))
    _check("S", S, torch.float32, (N, H, dk, dv))
    if out is None:
        out = torch.empty((N, H, dv), dtype=q.dtype, device=q.device)
    _check("out", out, q.dtype, (N, H, dv))
    rc = lib().kda_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S),
                               _ptr(out), N, H, dk, dv, dt, _stream(stream))
    if rc != KDA_OK:
        raise KdaError("kda_decode_step", rc)
    return out


def kda_decode_tokens(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor,
                      beta: torch.Tensor, S: torch.Tensor, out: Optional[torch.Tensor] = None,
                      stream=None) -> torch.Tensor:
    """L consecutive KDA decode steps in one launch.  q, k [N,L,H,dk]; v [N,L,H,dv];
    g [N,L,H,dk] f32; beta [N,L,H] f32; S [N,H,dk,dv] f32, updated in place (state
    after the last token).  Returns out [N,L,H,dv]; identical to L kda_decode_step
    calls."""
    if q.dim() != 4:
        raise ValueError("q must be [N, L, H, dk]")
    N, L, H, dk = q.shape
    dv = v.shape[-1]
    dt = _DTYPES.get(q.dtype)
    if dt is None:
        raise ValueError(f"unsupported dtype {q.dtype}")
    _check("q", q)
    _check("k", k, q.dtype, (N, L, H, dk))
    _check("v", v, q.dtype, (N, L, H, dv))
    G = _decay_group(g, dk)
    _check("g", g, torch.float32, (N, L, H, dk // G))
    _check("beta", beta, torch.float32, (N, L, H))
    _check("S", S, torch.float32, (N, H, dk, dv))
    if out is None:
        out = torch.empty((N, L, H, dv), dtype=q.dtype, device=q.device)
    _check("out", out, q.dtype, (N, L, H, dv))
    if G == 1:
        rc = lib().kda_decode_tokens(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S),
                                     _ptr(out), N, L, H, dk, dv, dt, _stream(stream))
    else:
        rc = lib().kda_decode_tokens_grouped(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                             _ptr(S), _ptr(out), N, L, H, dk, dv, G, dt,
                                             _stream(stream))
    if rc != KDA_OK:
        raise KdaError("kda_decode_tokens", rc)
    return out


def kda_decode_chunk(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor,
                     beta: torch.Tensor, S: torch.Tensor, out: Optional[torch.Tensor] = None,
                     stream=None) -> torch.Tensor:
    """L <= 16 tokens per (sequence, head) as one chunk of the chunked form on the tensor
    cores (bf16, dk = dv = 128).  Same layout and in-place S update as kda_decode_tokens;
    equal to L single steps up to the tensor-core rounding.  Returns out [N,L,H,dv]."""
    if q.dim() != 4:
        raise ValueError("q must be [N, L, H, dk]")
    N, L, H, dk = q.shape
    dv = v.shape[-1]
    dt = _DTYPES.get(q.dtype)
    if dt is None:
        raise ValueError(f"unsupported dtype {q.dtype}")
    _check("q", q)
    _check("k", k, q.dtype, (N, L, H, dk))
    _check("v", v, q.dtype, (N, L, H, dv))
    _check("g", g, torch.float32, (N, L, H, dk))
    _check("beta", beta, torch.float32, (N, L, H))
    _check("S", S, torch.float32, (N, H, dk, dv))
    if out is None:
        out = torch.empty((N, L, H, dv), dtype=q.dtype, device=q.device)
    _check("out", out, q.dtype, (N, L, H, dv))
    rc = lib().kda_decode_chunk(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S),
                                _ptr(out), N, L, H, dk, dv, dt, _stream(stream))
    if rc != KDA_OK:
        raise KdaError("kda_decode_chunk", rc)
    return out
