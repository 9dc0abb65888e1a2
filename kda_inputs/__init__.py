"""Seeded synthetic inputs for KDA (Kimi Delta Attention) prefill and decode.

This module is shared by the tests, the benchmark and the oracle's callers.  It
draws random tensors and prepares them the way a KDA layer's caller would
(L2-normalised q/k, q scaled by dk^-1/2, log-decay g <= 0, beta in (0, 1)); it
holds none of the delta-rule arithmetic itself.

Every tensor is produced on the CPU with a ``torch.Generator`` seeded per
workload, then rounded to its storage dtype.  Both the CUDA path and the oracle
consume exactly these rounded values (the oracle upcasts them to float64).

Workload shapes follow the models described on the source pages:
  * "Inside Kimi" / miniKimiK3 model card: 8 KDA heads x 64, rows of 256-512
    tokens (Architecture table, Training details table);
  * Mini-K3-1H model card: 12 heads x 128, 8K-token rows (Configuration list;
    "8K row length" paragraph of the Mamba-2 ablation card);
  * Kimi-K3-Tiny-L13 model card: 96 KDA heads x 128 ("What is preserved" table).

Distributions (N(mu, s): s is the standard deviation):
  * q, k ~ N(0, 1), L2-normalised per (token, head) over dk; q *= dk^-1/2.
  * v ~ N(0, 1).
  * decay "logsigmoid": g = log(sigmoid(x)), x ~ N(3, 1), per channel.
  * decay "alog": g = -exp(a_h) * softplus(u + dt_bias), a_h ~ U(-2, 0) per
    head, dt_bias ~ N(0, 0.5) per (head, channel), u ~ N(0, 1) per
    (token, head, channel)  (the A_log / dt_bias parameterisation the
    Kimi-K3-Tiny-L13 card mentions for its real KDA weights).
  * beta = sigmoid(N(0, 1)).
  * initial state, where used: N(0, 0.02), float32, layout [Nseq, H, dk, dv].
  * fused prep workloads (make_fused_prefill): raw q, k projections ~ N(0, 1)
    (not normalised), convolution taps ~ N(0, 0.5) of shape [H, dk, W], output
    gate pre-activations ~ N(0, 1).
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch

__all__ = [
    "PrefillSpec", "DecodeSpec", "PREFILL_SPECS", "DECODE_SPECS",
    "make_prefill", "make_fused_prefill", "make_decode", "doc_lengths", "spec_by_name",
    "strong_decay", "STRONG_DECAY_KINDS",
]


@dataclasses.dataclass(frozen=True)
class PrefillSpec:
    name: str
    B: int                 # batch rows (fixed length) or number of documents (varlen)
    T: int                 # tokens per row (fixed) or total packed tokens (varlen)
    H: int
    dk: int
    dv: int
    dtype: str             # "bf16" or "f32": storage dtype of q, k, v and out
    decay: str             # "logsigmoid" or "alog"
    seed: int
    h0: bool = False       # random initial state ~ N(0, 0.02)
    varlen: bool = False   # packed documents with cu_seqlens
    doc_min: int = 128
    doc_max: int = 4096
    desc: str = ""


@dataclasses.dataclass(frozen=True)
class DecodeSpec:
    name: str
    N: int
    H: int
    dk: int
    dv: int
    steps: int
    dtype: str
    decay: str
    seed: int
    desc: str = ""


# The workloads: four prefill shapes, the headline prefill shape, the decode shape.
PREFILL_SPECS = {
    "fp32_t256": PrefillSpec("fp32_t256", B=1, T=256, H=2, dk=64, dv=64, dtype="f32",
                        decay="logsigmoid", seed=0,
                        desc="fp32 KDA forward, B=1 T=256 H=2 d=64"),
    "b16_t512_d64": PrefillSpec("b16_t512_d64", B=16, T=512, H=8, dk=64, dv=64, dtype="bf16",
                        decay="logsigmoid", seed=1,
                        desc="miniKimiK3-shaped prefill, B=16 T=512 H=8 d=64"),
    "packed_16k": PrefillSpec("packed_16k", B=0, T=16384, H=12, dk=128, dv=128, dtype="bf16",
                        decay="alog", seed=2, varlen=True,
                        desc="Mini-K3-1H-shaped packed varlen prefill, 16384 tokens, "
                             "docs ~ U[128, 4096], H=12 d=128"),
    "t32k_h96": PrefillSpec("t32k_h96", B=1, T=32768, H=96, dk=128, dv=128, dtype="bf16",
                        decay="alog", seed=3, h0=True,
                        desc="Kimi-K3-width long prefill, B=1 T=32768 H=96 d=128, h0 ~ N(0,0.02)"),
    "t8k_h12": PrefillSpec("t8k_h12", B=1, T=8192, H=12, dk=128, dv=128, dtype="bf16",
                          decay="alog", seed=100,
                          desc="headline prefill, B=1 T=8192 H=12 d=128 bf16"),
}

DECODE_SPECS = {
    "decode_n256_h96": DecodeSpec("decode_n256_h96", N=256, H=96, dk=128, dv=128, steps=16, dtype="bf16",
                       decay="alog", seed=4,
                       desc="recurrent decode, N=256 x 16 tokens, H=96 d=128, "
                            "fp32 state ~ N(0,0.02) (1.61 GB)"),
}


def spec_by_name(name: str):
    if name in PREFILL_SPECS:
        return PREFILL_SPECS[name]
    return DECODE_SPECS[name]


def _torch_dtype(dtype: str) -> torch.dtype:
    return {"bf16": torch.bfloat16, "f32": torch.float32}[dtype]


def doc_lengths(total: int, lo: int, hi: int, gen: torch.Generator) -> list[int]:
    """Document lengths drawn uniformly from [lo, hi] until they reach ``total``;
    the last one is cut so the lengths sum to exactly ``total``."""
    lens: list[int] = []
    acc = 0
    while acc < total:
        n = int(torch.randint(lo, hi + 1, (1,), generator=gen).item())
        n = min(n, total - acc)
        lens.append(n)
        acc += n
    return lens


def _unit_rows(x: torch.Tensor) -> torch.Tensor:
    # L2 normalisation over the last axis (caller-side input preparation).
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-12)


def _decay(shape_tok: tuple, H: int, dk: int, decay: str, gen: torch.Generator) -> torch.Tensor:
    """Log-decay g <= 0 of shape shape_tok + (H, dk), float32."""
    if decay == "logsigmoid":
        x = torch.randn(*shape_tok, H, dk, generator=gen) + 3.0
        return torch.nn.functional.logsigmoid(x)
    if decay == "alog":
        a = torch.rand(H, generator=gen) * 2.0 - 2.0                 # U(-2, 0)
        dt_bias = torch.randn(H, dk, generator=gen) * 0.5             # N(0, 0.5)
        u = torch.randn(*shape_tok, H, dk, generator=gen)             # N(0, 1)
        return -torch.exp(a)[:, None] * torch.nn.functional.softplus(u + dt_bias)
    raise ValueError(decay)


def _qkvb(shape_tok: tuple, H: int, dk: int, dv: int, gen: torch.Generator):
    q = _unit_rows(torch.randn(*shape_tok, H, dk, generator=gen)) * (dk ** -0.5)
    k = _unit_rows(torch.randn(*shape_tok, H, dk, generator=gen))
    v = torch.randn(*shape_tok, H, dv, generator=gen)
    beta = torch.sigmoid(torch.randn(*shape_tok, H, generator=gen))
    return q, k, v, beta


def make_prefill(spec: PrefillSpec | str, *, T: Optional[int] = None, B: Optional[int] = None,
                 H: Optional[int] = None, seed: Optional[int] = None,
                 doc_lens: Optional[list[int]] = None) -> dict:
    """Inputs for one ``kda_chunk_fwd`` call, as CPU tensors in storage dtype.

    Keyword overrides shrink a workload (same distributions) for tests.
    Returns a dict with q, k, v ([B,T,H,dk|dv], storage dtype), g ([B,T,H,dk] f32),
    beta ([B,T,H] f32), h0 ([Nseq,H,dk,dv] f32 or None), cu_seqlens (int32
    [Nseq+1] or None) and the sizes.  For varlen workloads B in the tensors is 1.
    """
    if isinstance(spec, str):
        spec = PREFILL_SPECS[spec]
    T = spec.T if T is None else T
    H = spec.H if H is None else H
    seed = spec.seed if seed is None else seed
    gen = torch.Generator().manual_seed(seed)
    dk, dv = spec.dk, spec.dv
    cu = None
    if spec.varlen or doc_lens is not None:
        if doc_lens is None:
            doc_lens = doc_lengths(T, spec.doc_min, spec.doc_max, gen)
        T = int(sum(doc_lens))
        cu = torch.zeros(len(doc_lens) + 1, dtype=torch.int32)
        cu[1:] = torch.cumsum(torch.tensor(doc_lens, dtype=torch.int64), 0).to(torch.int32)
        Bt, nseq = 1, len(doc_lens)
    else:
        Bt = spec.B if B is None else B
        nseq = Bt
    q, k, v, beta = _qkvb((Bt, T), H, dk, dv, gen)
    g = _decay((Bt, T), H, dk, spec.decay, gen)
    h0 = None
    if spec.h0:
        h0 = torch.randn(nseq, H, dk, dv, generator=gen) * 0.02
    dt = _torch_dtype(spec.dtype)
    return dict(q=q.to(dt).contiguous(), k=k.to(dt).contiguous(), v=v.to(dt).contiguous(),
                g=g.float().contiguous(), beta=beta.float().contiguous(),
                h0=None if h0 is None else h0.float().contiguous(),
                cu_seqlens=cu, B=nseq, T=T, H=H, dk=dk, dv=dv, dtype=spec.dtype,
                name=spec.name)


def make_fused_prefill(spec: PrefillSpec | str, *, W: int = 4, gate: bool = True,
                       T: Optional[int] = None, B: Optional[int] = None, H: Optional[int] = None,
                       seed: Optional[int] = None, doc_lens: Optional[list[int]] = None) -> dict:
    """Inputs for one ``kda_chunk_fwd_fused`` call: ``make_prefill``'s tensors
    (v, g, beta, h0, cu_seqlens) plus raw q, k projections (q_raw, k_raw, storage
    dtype), convolution taps conv_q, conv_k ([H, dk, W] f32) and, with ``gate``,
    the gate pre-activations gate ([B, T, H, dv], storage dtype)."""
    if isinstance(spec, str):
        spec = PREFILL_SPECS[spec]
    x = make_prefill(spec, T=T, B=B, H=H, seed=seed, doc_lens=doc_lens)
    gen = torch.Generator().manual_seed((spec.seed if seed is None else seed) + 7919)
    dt = _torch_dtype(spec.dtype)
    Bt, Tt, Hh, dk = x["q"].shape
    dv = x["v"].shape[-1]
    x["q_raw"] = torch.randn(Bt, Tt, Hh, dk, generator=gen).to(dt).contiguous()
    x["k_raw"] = torch.randn(Bt, Tt, Hh, dk, generator=gen).to(dt).contiguous()
    x["conv_q"] = (torch.randn(Hh, dk, W, generator=gen) * 0.5).float().contiguous()
    x["conv_k"] = (torch.randn(Hh, dk, W, generator=gen) * 0.5).float().contiguous()
    x["gate"] = (torch.randn(Bt, Tt, Hh, dv, generator=gen).to(dt).contiguous() if gate
                 else None)
    x["W"] = W
    return x


def make_decode(spec: DecodeSpec | str, *, N: Optional[int] = None, H: Optional[int] = None,
                steps: Optional[int] = None, seed: Optional[int] = None) -> dict:
    """Inputs for ``steps`` consecutive ``kda_decode_step`` calls, CPU tensors.

    q, k: [steps, N, H, dk]; v: [steps, N, H, dv] (storage dtype);
    g: [steps, N, H, dk] f32; beta: [steps, N, H] f32; S0: [N, H, dk, dv] f32.
    """
    if isinstance(spec, str):
        spec = DECODE_SPECS[spec]
    N = spec.N if N is None else N
    H = spec.H if H is None else H
    steps = spec.steps if steps is None else steps
    seed = spec.seed if seed is None else seed
    gen = torch.Generator().manual_seed(seed)
    dk, dv = spec.dk, spec.dv
    S0 = torch.randn(N, H, dk, dv, generator=gen) * 0.02
    q, k, v, beta = _qkvb((steps, N), H, dk, dv, gen)
    g = _decay((steps, N), H, dk, spec.decay, gen)
    dt = _torch_dtype(spec.dtype)
    return dict(q=q.to(dt).contiguous(), k=k.to(dt).contiguous(), v=v.to(dt).contiguous(),
                g=g.float().contiguous(), beta=beta.float().contiguous(),
                S0=S0.float().contiguous(), N=N, H=H, dk=dk, dv=dv, steps=steps,
                dtype=spec.dtype, name=spec.name)


STRONG_DECAY_KINDS = ("channels", "spikes", "both")


def strong_decay(g: torch.Tensor, kind: str, *, token_dim: int, seed: int = 0) -> torch.Tensor:
    """A copy of the log-decay ``g`` (float32, key channels on the last axis, tokens on
    ``token_dim``) with strong and complete-forgetting decay planted in it.

    These are the decay inputs at the edge of any factoring of exp(G_r - G_i)
    through per-block reference points: a 16-token block whose cumulative log-decay
    on a channel falls far below -80.

      "channels": key channels 1, 5, dk/2 + 3 and dk - 2 of every head decay by
                  g ~ U(-6.5, -5.5) at every token (about -96 over 16 tokens);
      "spikes":   isolated tokens whose gate closes on every channel: g = -20 at
                  tokens t = 5 (mod 23) and g = -1e4 at t = 11 (mod 37) (alpha = 0
                  in float32: complete forgetting), plus g = -1e4 on every other
                  channel at t = 2 (mod 29) -- all of them inside 16-token blocks,
                  not only at their first rows;
      "both":     the two together.
    Where two rules hit one element the later one in this list wins.
    """
    if kind not in STRONG_DECAY_KINDS:
        raise ValueError(kind)
    out = g.clone()
    dk = g.shape[-1]
    nt = g.shape[token_dim]
    gen = torch.Generator().manual_seed(seed + 104729)
    tok = torch.arange(nt)

    def at_tokens(mask: torch.Tensor) -> torch.Tensor:
        # index tuple selecting the tokens in ``mask`` along token_dim
        idx = [slice(None)] * g.dim()
        idx[token_dim] = mask.nonzero().flatten()
        return tuple(idx)

    if kind in ("channels", "both"):
        chans = sorted({1, 5, dk // 2 + 3, dk - 2})
        noise = torch.rand(*g.shape[:-1], len(chans), generator=gen)
        out[..., chans] = -6.5 + noise
    if kind in ("spikes", "both"):
        out[at_tokens(tok % 23 == 5)] = -20.0
        out[at_tokens(tok % 37 == 11)] = -1.0e4
        sel = list(at_tokens(tok % 29 == 2))
        sub = out[tuple(sel)]
        sub[..., 0::2] = -1.0e4
        out[tuple(sel)] = sub
    return out.contiguous()
