"""Shared helpers for the GPU parity tests: run the CUDA path and the oracle on the
same seeded inputs and compare them by the relative error
max|x - x_ref| / max|x_ref| (computed separately for the output and the state)."""
from __future__ import annotations

import numpy as np
import torch

# Tolerances on max|x - x_ref| / max|x_ref|, for out and for the final state.
TOL = {"bf16": 1e-2, "f32": 1e-4}


def rel_err(x, ref) -> float:
    x = x.detach().double().cpu().numpy() if hasattr(x, "detach") else np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.abs(ref).max()
    if den == 0:
        return float(np.abs(x).max())
    return float(np.abs(x - ref).max() / den)


def to_dev(x: dict, device="cuda") -> dict:
    return {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


def gpu_prefill(x: dict, with_h0=True, out_state=True):
    import gated_delta_rule_74_b200 as kda
    d = to_dev(x)
    out, hT = kda.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"],
                                h0=d["h0"] if with_h0 else None, cu_seqlens=d["cu_seqlens"],
                                output_final_state=out_state)
    torch.cuda.synchronize()
    return out, hT


def oracle_prefill(x: dict, heads=None, with_h0=True):
    import oracle
    return oracle.prefill(x["q"], x["k"], x["v"], x["g"], x["beta"],
                          x["h0"] if with_h0 else None, x["cu_seqlens"], heads=heads)
