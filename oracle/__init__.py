"""KDA oracle: a plain, slow, float64 CPU implementation of Kimi Delta Attention.

TEST INFRASTRUCTURE ONLY.  The tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference legs are the only callers.  The CUDA path
(``gated_delta_rule_74_b200``) never imports this package and shares no code
with it; the only module both sides use is ``kda_inputs`` (seeded random
inputs, none of the method's arithmetic).

Contents
  * ``prefill`` / ``decode``: ctypes front end of ``kda_oracle.cpp``, the
    token-by-token float64 recurrence
        S_t = (I - beta_t k_t k_t^T) Diag(exp(g_t)) S_{t-1} + beta_t k_t v_t^T,
        o_t = S_t^T q_t
    (miniKimiK3 model card, Architecture, "Kimi Delta Attention" bullet), with
    the state reset to each document's own initial state at every cu_seqlens
    boundary (Mini-K3-1H-mamba2 model card, packed-document paragraph).
  * ``reference.recurrence_literal``: the same recurrence in numpy with the
    dk x dk factor (I - beta k k^T) materialised, for tiny inputs.
  * ``reference.chunked``: the chunked (WY / UT transform) form of the same
    recurrence in float64 numpy, for checking the chunked algebra the GPU
    kernels implement ("trains through a chunked parallel form", same bullet).

  * ``prefill_fused`` (with ``short_conv``, ``l2_normalize``, ``output_gate``):
    the input prep and output gate around KDA that the Mini-K3-1H v2 family
    cards name (short convolutions, output gates) but do not define; the reading
    taken is stated in ``prefill_fused``.
  * ``backward``: float64 reverse-mode gradients of the recurrence.

Pins: tests/test_oracle.py checks these routines against closed forms,
invariants, a hand-worked example (tests/golden/) and brute force.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

from . import reference  # noqa: F401  (numpy routines)

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.cpp")
_SO = os.path.join(_HERE, "libkda_oracle.so")
_lib = None
_lock = threading.Lock()

__all__ = ["build", "prefill", "decode", "backward", "prefill_fused", "short_conv",
           "l2_normalize", "output_gate", "max_threads", "reference"]


def build(force: bool = False) -> str:
    """Compile kda_oracle.cpp into libkda_oracle.so next to it (no fast-math)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        cmd = ["g++", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
               "-shared", "-fPIC", "-std=c++17", _SRC, "-o", _SO + ".tmp"]
        subprocess.run(cmd, check=True)
        os.replace(_SO + ".tmp", _SO)
    return _SO


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_SO)
            dp = ctypes.POINTER(ctypes.c_double)
            lib.kda_oracle_prefill.argtypes = [dp, dp, dp, dp, dp, dp,
                                               ctypes.POINTER(ctypes.c_int32), dp, dp,
                                               ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                               ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                               ctypes.c_int, ctypes.c_int]
            lib.kda_oracle_prefill.restype = ctypes.c_int
            lib.kda_oracle_decode.argtypes = [dp, dp, dp, dp, dp, dp, dp,
                                              ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                              ctypes.c_int, ctypes.c_longlong,
                                              ctypes.c_longlong, ctypes.c_int]
            lib.kda_oracle_decode.restype = ctypes.c_int
            lib.kda_oracle_backward.argtypes = ([dp] * 6 + [ctypes.POINTER(ctypes.c_int32)] +
                                                [dp] * 8 + [ctypes.c_int] * 8)
            lib.kda_oracle_backward.restype = ctypes.c_int
            lib.kda_oracle_max_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def max_threads() -> int:
    return int(_load().kda_oracle_max_threads())


def _f64(x) -> np.ndarray:
    """Exact upcast of a torch tensor (bf16/f32) or array to contiguous float64."""
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def expand_decay_groups(g, dk: int):
    """Grouped decay (one log-decay per group of G = dk / g.shape[-1] consecutive key
    channels, the "decay-g64" family card's decay-granularity variant): channel c
    decays by exp(g[..., c // G]).  Returns the per-channel [..., dk] float64 array."""
    g = _f64(g)
    n = g.shape[-1]
    if n == dk:
        return g
    if n < 1 or dk % n != 0:
        raise ValueError(f"g's last dimension {n} does not divide dk = {dk}")
    return np.ascontiguousarray(np.repeat(g, dk // n, axis=-1))


def prefill(q, k, v, g, beta, h0=None, cu_seqlens=None, heads=None, nthreads: int = 0):
    """Float64 KDA prefill by recurrence.

    q, k [B,T,H,dk]; v [B,T,H,dv]; g [B,T,H,dk] (or [B,T,H,dk/G]: one decay per group
    of G key channels, see expand_decay_groups); beta [B,T,H]; h0 [Nseq,H,dk,dv]
    or None; cu_seqlens int [Nseq+1] or None (then tensors are [1,T,H,*]).
    ``heads``: optional (lo, hi) range; only those heads are computed and returned.
    Returns (out [B,T,H',dv], hT [Nseq,H',dk,dv]) as float64 numpy arrays.
    """
    g = expand_decay_groups(g, q.shape[-1])
    if heads is not None:
        lo, hi = heads
        q, k, v, g, beta = (x[:, :, lo:hi] for x in (q, k, v, g, beta))
        if h0 is not None:
            h0 = h0[:, lo:hi]
    q, k, v, g, beta, h0 = (_f64(x) for x in (q, k, v, g, beta, h0))
    Bt, T, H, dk = q.shape
    dv = v.shape[-1]
    cu = None
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(cu_seqlens.cpu() if hasattr(cu_seqlens, "cpu")
                                             else cu_seqlens), dtype=np.int32)
        nseq = cu.shape[0] - 1
        if Bt != 1:
            raise ValueError("packed (cu_seqlens) inputs must have B == 1 in the tensors")
    else:
        nseq = Bt
    out = np.zeros((Bt, T, H, dv), dtype=np.float64)
    hT = np.zeros((nseq, H, dk, dv), dtype=np.float64)
    rc = _load().kda_oracle_prefill(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0),
        None if cu is None else cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
        _ptr(out), _ptr(hT), nseq, T, H, dk, dv, 0, H, int(nthreads))
    if rc != 0:
        raise ValueError(f"kda_oracle_prefill rejected its arguments (rc={rc})")
    return out, hT


def decode(q, k, v, g, beta, S, nthreads: int = 0):
    """One float64 KDA decode step.  q,k [N,H,dk]; v [N,H,dv]; g [N,H,dk];
    beta [N,H]; S [N,H,dk,dv].  Returns (out [N,H,dv], S_new) as float64 arrays
    (S is copied, not modified).  g may be grouped ([N,H,dk/G], expand_decay_groups)."""
    g = expand_decay_groups(g, q.shape[-1])
    q, k, v, g, beta = (_f64(x) for x in (q, k, v, g, beta))
    S = _f64(S).copy()
    N, H, dk = q.shape
    dv = v.shape[-1]
    out = np.zeros((N, H, dv), dtype=np.float64)
    rc = _load().kda_oracle_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                   _ptr(S), _ptr(out), N, H, dk, dv, 0, N * H,
                                   int(nthreads))
    if rc != 0:
        raise ValueError(f"kda_oracle_decode rejected its arguments (rc={rc})")
    return out, S


def backward(q, k, v, g, beta, dout, h0=None, dhT=None, cu_seqlens=None, heads=None,
             nthreads: int = 0):
    """Float64 gradients of L = sum(out * dout) + sum(hT * dhT) for the prefill
    (reverse-mode differentiation of the recurrence; kda_oracle.cpp).

    Shapes as in ``prefill``; dout [B,T,H,dv]; dhT [Nseq,H,dk,dv] or None.
    Returns a dict of float64 arrays dq, dk, dv, dg, dbeta, dh0 (dg has g's
    per-channel shape [B,T,H,dk]; for grouped g sum it over each group).
    """
    if heads is not None:
        lo, hi = heads
        q, k, v, g, beta, dout = (x[:, :, lo:hi] for x in (q, k, v, g, beta, dout))
        if h0 is not None:
            h0 = h0[:, lo:hi]
        if dhT is not None:
            dhT = dhT[:, lo:hi]
    g = expand_decay_groups(g, q.shape[-1])
    q, k, v, g, beta, h0, dout, dhT = (_f64(x) for x in (q, k, v, g, beta, h0, dout, dhT))
    Bt, T, H, dk = q.shape
    dv = v.shape[-1]
    cu = None
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(cu_seqlens.cpu() if hasattr(cu_seqlens, "cpu")
                                             else cu_seqlens), dtype=np.int32)
        nseq = cu.shape[0] - 1
    else:
        nseq = Bt
    res = {n: np.zeros(x.shape, dtype=np.float64) for n, x in
           (("dq", q), ("dk", k), ("dv", v), ("dg", g), ("dbeta", beta))}
    res["dh0"] = np.zeros((nseq, H, dk, dv), dtype=np.float64)
    rc = _load().kda_oracle_backward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0),
        None if cu is None else cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
        _ptr(dout), _ptr(dhT), _ptr(res["dq"]), _ptr(res["dk"]), _ptr(res["dv"]),
        _ptr(res["dg"]), _ptr(res["dbeta"]), _ptr(res["dh0"]), nseq, T, H, dk, dv, 0, H,
        int(nthreads))
    if rc != 0:
        raise ValueError(f"kda_oracle_backward rejected its arguments (rc={rc})")
    return res


def _doc_ranges(T: int, Bt: int, cu_seqlens):
    """(batch row, first token, end token) of every document."""
    if cu_seqlens is None:
        return [(b, 0, T) for b in range(Bt)]
    cu = np.asarray(cu_seqlens.cpu() if hasattr(cu_seqlens, "cpu") else cu_seqlens,
                    dtype=np.int64)
    return [(0, int(cu[d]), int(cu[d + 1])) for d in range(cu.shape[0] - 1)]


def short_conv(x, w, cu_seqlens=None):
    """Causal per-channel convolution over tokens, restarting at every document:
    y_t[h, i] = sum_{j<W} w[h, i, j] * x_{t-W+1+j}[h, i], with x = 0 before the
    document's first token (Mini-K3-1H-mamba2 card: convolution history is reset
    at every document boundary).  x [B,T,H,d]; w [H,d,W].  float64 result."""
    x, w = _f64(x), _f64(w)
    Bt, T = x.shape[:2]
    W = w.shape[-1]
    y = np.zeros_like(x)
    for b, t0, t1 in _doc_ranges(T, Bt, cu_seqlens):
        for t in range(t0, t1):
            for j in range(W):
                src = t - (W - 1) + j
                if src >= t0:
                    y[b, t] += w[:, :, j] * x[b, src]
    return y


def l2_normalize(x, eps: float = 1e-12):
    """x / max(||x||_2, eps) over the last axis (per token and head)."""
    x = _f64(x)
    n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True))
    return x / np.maximum(n, eps)


def output_gate(o, z):
    """o * sigmoid(z), elementwise (the output gate of the family cards)."""
    o, z = _f64(o), _f64(z)
    return o / (1.0 + np.exp(-z))


def prefill_fused(q_raw, k_raw, v, g, beta, conv_q=None, conv_k=None, gate=None, h0=None,
                  cu_seqlens=None, heads=None, nthreads: int = 0):
    """KDA prefill with its input prep and output gate, in float64.

    Reading (the pages name short convolutions, q/k normalisation and output
    gates without defining them): q = dk^-1/2 * l2_normalize(short_conv(q_raw, conv_q)),
    k = l2_normalize(short_conv(k_raw, conv_k)), v unchanged; with conv_q = conv_k =
    None, q = q_raw and k = k_raw.  out = output_gate(o, gate) when gate is given.
    Returns (out, hT) as ``prefill`` does (``heads`` selects a head range).
    """
    if heads is not None:
        lo, hi = heads
        q_raw, k_raw, v, g, beta = (x[:, :, lo:hi] for x in (q_raw, k_raw, v, g, beta))
        conv_q = None if conv_q is None else conv_q[lo:hi]
        conv_k = None if conv_k is None else conv_k[lo:hi]
        gate = None if gate is None else gate[:, :, lo:hi]
        h0 = None if h0 is None else h0[:, lo:hi]
    if (conv_q is None) != (conv_k is None):
        raise ValueError("give both conv_q and conv_k, or neither")
    if conv_q is not None:
        dk = q_raw.shape[-1]
        q = l2_normalize(short_conv(q_raw, conv_q, cu_seqlens)) / np.sqrt(dk)
        k = l2_normalize(short_conv(k_raw, conv_k, cu_seqlens))
    else:
        q, k = _f64(q_raw), _f64(k_raw)
    out, hT = prefill(q, k, v, g, beta, h0, cu_seqlens, nthreads=nthreads)
    if gate is not None:
        out = output_gate(out, gate)
    return out, hT
