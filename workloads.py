"""Seeded synthetic inputs for the gated delta-rule prefill and decode paths.

This module is shared by the tests, ``bench.py`` and ``__graft_entry__.smoke``.
It only draws and shapes random inputs; it holds none of the recurrence's
arithmetic.  The distributions follow the layer the pages describe:

* the Qwen2.5-0.5B KDA graft ("kda-graft", section "Идея и архитектура"):
  14 heads of dimension 64, an alpha gate initialised with bias +5 so that
  sigmoid(5) ~ 0.993, and an fp32 recurrent state;
* the Gated DeltaNet hybrids ("Modele hybrydowe: co Gated DeltaNet zastępuje
  w cache KV", sections "Atencja liniowa" and "Gated DeltaNet: dodaj zanik"):
  head dimension 128 and contexts up to 262K tokens.

Every tensor is drawn in fp32 from a CPU (or CUDA) ``torch.Generator`` seeded
per workload, normalised where stated, then cast once to the compute dtype.
Both sides of a parity test receive exactly those bits.

Layouts (token-major, packed over sequences by ``cu_seqlens``):
  q, k     [T_tot, H, d_k]     v        [T_tot, H, d_v]
  beta     [T_tot, H] fp32     log_a    [T_tot, H, d_k] or [T_tot, H] (scalar gate)
  state    [N, H, d_v, d_k] fp32 (row = value channel, column = key channel)
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Optional

import torch


@dataclass(frozen=True)
class PrefillWorkload:
    name: str
    seed: int
    n_heads: int
    d_k: int
    d_v: int
    lengths: Optional[tuple] = None      # fixed lengths; None -> drawn (varlen)
    n_seqs: int = 1
    len_range: Optional[tuple] = None    # inclusive uniform range for varlen
    qkv_dtype: torch.dtype = torch.bfloat16
    scalar_decay: bool = False
    log_a_mu: float = 5.0                # log_a = logsigmoid(N(mu, sd))
    log_a_sd: float = 1.0
    log_a_clamp: Optional[tuple] = None  # (lo, hi) applied after logsigmoid
    init_std: float = 0.0                # 0 -> zero initial state
    snap_interval: int = 0
    scale: float = 1.0


@dataclass(frozen=True)
class DecodeWorkload:
    name: str
    seed: int
    batch: int
    n_heads: int
    d_k: int
    d_v: int
    steps: int
    qkv_dtype: torch.dtype = torch.bfloat16
    scalar_decay: bool = False
    log_a_mu: float = 5.0
    log_a_sd: float = 1.0
    init_std: float = 0.1
    scale: float = 1.0


# The five workloads the method is measured on.  Seeds are 1000 + index.
TINY_KDA = PrefillWorkload("tiny_kda_H2_T256_d64_f32", 1001, 2, 64, 64,
                           lengths=(256,), qkv_dtype=torch.float32)
GRAFT_LAYER = PrefillWorkload("graft_layer_H14_T8192_d64_bf16", 1002, 14, 64, 64,
                              lengths=(8192,))
DECODE = DecodeWorkload("decode_B256_H14_d64_1024steps", 1003, 256, 14, 64, 64, 1024)
GDN_LONG = PrefillWorkload("gdn_long_H16_T65536_d128_scalar_snap4096", 1004, 16, 128, 128,
                           lengths=(65536,), scalar_decay=True, log_a_mu=4.0,
                           log_a_sd=1.5, snap_interval=4096)
VARLEN = PrefillWorkload("varlen_N32_H32_d128_L1024to16384", 1005, 32, 128, 128,
                         n_seqs=32, len_range=(1024, 16384), log_a_mu=3.0,
                         log_a_sd=2.0, log_a_clamp=(-5.0, 0.0), init_std=0.1)

PREFILL_WORKLOADS = {w.name: w for w in (TINY_KDA, GRAFT_LAYER, GDN_LONG, VARLEN)}


@dataclass(frozen=True)
class DraftWorkload:
    """Speculative decoding on the decode workload's sequences: each round
    drafts K tokens per sequence from the live state, then accepts a number
    of them drawn uniformly from 0 .. K."""
    name: str
    seed: int
    decode: DecodeWorkload      # sizes and distributions of state and tokens
    draft_tokens: int
    rounds: int


SPEC_DRAFT = DraftWorkload("spec_draft_B256_H14_d64_K4", 1006, DECODE, 4, 16)

# Raw projections of the graft layer's shape for the input activations: the
# gates come out distributed as the graft layer's (beta = sigmoid(N(0, 1)),
# log a = logsigmoid(5 + N(0, 1)) with the page's bias +5).
PREPROCESS = replace(GRAFT_LAYER, name="preprocess_graft_layer_H14_T8192_d64_bf16", seed=1007)

# Smaller cases of the d 128 workloads (same distributions) for ncu captures,
# which replay each captured launch many times: a few GB on the device at most.
PROFILE_CASES = {w.name: w for w in (
    replace(GDN_LONG, name="gdn_H16_T16384_d128_scalar", lengths=(16384,), snap_interval=0),
    replace(VARLEN, name="varlen_N4_H32_d128_L1024to16384", n_seqs=4),
)}


def shrink(w: PrefillWorkload, **kw) -> PrefillWorkload:
    """Same distributions, other sizes (for fast parity cases)."""
    return replace(w, **kw)


def _l2norm(x: torch.Tensor) -> torch.Tensor:
    # Per (token, head) normalisation in fp32; Gaussian rows never vanish.
    return x / x.norm(dim=-1, keepdim=True)


def _draw_lengths(w: PrefillWorkload, gen: torch.Generator) -> list:
    if w.lengths is not None:
        return list(w.lengths)
    lo, hi = w.len_range
    return torch.randint(lo, hi + 1, (w.n_seqs,), generator=gen).tolist()


def cu_seqlens_of(lengths) -> torch.Tensor:
    cu = [0]
    for n in lengths:
        cu.append(cu[-1] + int(n))
    return torch.tensor(cu, dtype=torch.int32)


def make_prefill_inputs(w: PrefillWorkload, device="cpu", lengths=None,
                        draw_device=None) -> dict:
    """Draw one batch of prefill inputs.

    ``draw_device`` selects where the random numbers are drawn ("cpu" by
    default: bit-identical on every machine; "cuda" for multi-GB workloads).
    The result lives on ``device``.
    """
    draw_device = draw_device or "cpu"
    gen = torch.Generator(device=draw_device)
    gen.manual_seed(w.seed)
    if lengths is None:
        # lengths always come from a CPU generator so they never depend on device
        lgen = torch.Generator().manual_seed(w.seed)
        lengths = _draw_lengths(w, lgen)
    lengths = [int(n) for n in lengths]
    T = sum(lengths)
    H, dk, dv = w.n_heads, w.d_k, w.d_v
    f32 = dict(dtype=torch.float32, device=draw_device, generator=gen)
    q = _l2norm(torch.randn(T, H, dk, **f32)).to(w.qkv_dtype)
    k = _l2norm(torch.randn(T, H, dk, **f32)).to(w.qkv_dtype)
    v = torch.randn(T, H, dv, **f32).to(w.qkv_dtype)
    beta = torch.sigmoid(torch.randn(T, H, **f32))
    la_shape = (T, H) if w.scalar_decay else (T, H, dk)
    log_a = torch.nn.functional.logsigmoid(w.log_a_mu + w.log_a_sd * torch.randn(la_shape, **f32))
    if w.log_a_clamp is not None:
        log_a = log_a.clamp(*w.log_a_clamp)
    n = len(lengths)
    if w.init_std > 0:
        init = w.init_std * torch.randn(n, H, dv, dk, **f32)
    else:
        init = None
    out = dict(q=q, k=k, v=v, beta=beta.contiguous(), log_a=log_a.contiguous(),
               init_state=init, cu_seqlens=cu_seqlens_of(lengths), lengths=lengths,
               scalar_decay=w.scalar_decay, scale=w.scale, snap_interval=w.snap_interval)
    dev = torch.device(device)
    for key in ("q", "k", "v", "beta", "log_a", "init_state", "cu_seqlens"):
        if out[key] is not None:
            out[key] = out[key].to(dev).contiguous()
    return out


def make_decode_inputs(w: DecodeWorkload, steps: Optional[int] = None, device="cpu",
                       draw_device=None) -> dict:
    """Initial state plus ``steps`` fresh single-token inputs per sequence/head.

    Per-step tensors carry a leading step axis: q, k [S, B, H, d_k],
    v [S, B, H, d_v], beta [S, B, H], log_a [S, B, H, d_k] (or [S, B, H]).
    """
    steps = w.steps if steps is None else steps
    draw_device = draw_device or "cpu"
    gen = torch.Generator(device=draw_device)
    gen.manual_seed(w.seed)
    B, H, dk, dv = w.batch, w.n_heads, w.d_k, w.d_v
    f32 = dict(dtype=torch.float32, device=draw_device, generator=gen)
    state = w.init_std * torch.randn(B, H, dv, dk, **f32)
    q = _l2norm(torch.randn(steps, B, H, dk, **f32)).to(w.qkv_dtype)
    k = _l2norm(torch.randn(steps, B, H, dk, **f32)).to(w.qkv_dtype)
    v = torch.randn(steps, B, H, dv, **f32).to(w.qkv_dtype)
    beta = torch.sigmoid(torch.randn(steps, B, H, **f32))
    la_shape = (steps, B, H) if w.scalar_decay else (steps, B, H, dk)
    log_a = torch.nn.functional.logsigmoid(w.log_a_mu + w.log_a_sd * torch.randn(la_shape, **f32))
    out = dict(state=state, q=q, k=k, v=v, beta=beta, log_a=log_a,
               scalar_decay=w.scalar_decay, scale=w.scale)
    dev = torch.device(device)
    for key in ("state", "q", "k", "v", "beta", "log_a"):
        out[key] = out[key].to(dev).contiguous()
    return out



def make_draft_inputs(w: DraftWorkload, rounds: Optional[int] = None, device="cpu",
                      draw_device=None) -> dict:
    """Initial state plus ``rounds`` drafts of K tokens per sequence, drawn
    like the decode workload's tokens, and the accepted count per round and
    sequence.  q, k [R, B, K, H, d_k], v [R, B, K, H, d_v], beta [R, B, K, H],
    log_a [R, B, K, H, d_k] (or [R, B, K, H]), n_accept [R, B] int32 in 0 .. K.
    """
    d = w.decode
    R = w.rounds if rounds is None else rounds
    K = w.draft_tokens
    draw_device = draw_device or "cpu"
    gen = torch.Generator(device=draw_device)
    gen.manual_seed(w.seed)
    B, H, dk, dv = d.batch, d.n_heads, d.d_k, d.d_v
    f32 = dict(dtype=torch.float32, device=draw_device, generator=gen)
    state = d.init_std * torch.randn(B, H, dv, dk, **f32)
    q = _l2norm(torch.randn(R, B, K, H, dk, **f32)).to(d.qkv_dtype)
    k = _l2norm(torch.randn(R, B, K, H, dk, **f32)).to(d.qkv_dtype)
    v = torch.randn(R, B, K, H, dv, **f32).to(d.qkv_dtype)
    beta = torch.sigmoid(torch.randn(R, B, K, H, **f32))
    la_shape = (R, B, K, H) if d.scalar_decay else (R, B, K, H, dk)
    log_a = torch.nn.functional.logsigmoid(d.log_a_mu + d.log_a_sd * torch.randn(la_shape, **f32))
    n_accept = torch.randint(0, K + 1, (R, B), generator=gen, device=draw_device,
                             dtype=torch.int32)
    out = dict(state=state, q=q, k=k, v=v, beta=beta, log_a=log_a, n_accept=n_accept,
               scalar_decay=d.scalar_decay, scale=d.scale)
    dev = torch.device(device)
    for key in ("state", "q", "k", "v", "beta", "log_a", "n_accept"):
        out[key] = out[key].to(dev).contiguous()
    return out


def make_preprocess_inputs(w: PrefillWorkload, device="cpu", lengths=None, draw_device=None,
                           conv_noise: float = 0.1, gate_bias: float = 5.0) -> dict:
    """Raw per-head projections and parameters for the input activations.

    xq, xk, xv ~ N(0, 1) [T, H, d] (cast to the workload's dtype); conv taps
    [H d, 4] = the identity tap [0, 0, 0, 1] plus N(0, conv_noise); beta_raw ~
    N(0, 1) [T, H]; a_raw ~ N(0, 1) [T, H, d] (or [T, H]) with a bias of
    ``gate_bias`` per (head, channel) (or per head).
    """
    draw_device = draw_device or "cpu"
    gen = torch.Generator(device=draw_device)
    gen.manual_seed(w.seed)
    if lengths is None:
        lgen = torch.Generator().manual_seed(w.seed)
        lengths = _draw_lengths(w, lgen)
    lengths = [int(n) for n in lengths]
    T = sum(lengths)
    H, d = w.n_heads, w.d_k
    f32 = dict(dtype=torch.float32, device=draw_device, generator=gen)
    x = [torch.randn(T, H, d, **f32).to(w.qkv_dtype) for _ in range(3)]
    ident = torch.tensor([0.0, 0.0, 0.0, 1.0], device=draw_device)
    conv = [ident + conv_noise * torch.randn(H * d, 4, **f32) for _ in range(3)]
    beta_raw = torch.randn(T, H, **f32)
    a_raw = torch.randn((T, H) if w.scalar_decay else (T, H, d), **f32)
    a_bias = torch.full((H,) if w.scalar_decay else (H, d), gate_bias, device=draw_device)
    out = dict(xq=x[0], xk=x[1], xv=x[2], conv_q=conv[0], conv_k=conv[1], conv_v=conv[2],
               beta_raw=beta_raw, a_raw=a_raw, a_bias=a_bias, cu_seqlens=cu_seqlens_of(lengths),
               lengths=lengths, scalar_decay=w.scalar_decay)
    dev = torch.device(device)
    for key in ("xq", "xk", "xv", "conv_q", "conv_k", "conv_v", "beta_raw", "a_raw", "a_bias",
                "cu_seqlens"):
        out[key] = out[key].to(dev).contiguous()
    return out


def make_output_gate(T: int, H: int, d_v: int, dtype: torch.dtype, seed: int, device="cpu",
                     draw_device=None) -> dict:
    """Inputs of the output epilogue (RMSNorm and output gate, "kda-graft",
    section "Идея и архитектура"): a raw gate projection gate_raw [T, H, d_v]
    ~ N(0, 1) in the outputs' dtype and an RMSNorm weight [d_v] = 1 + N(0, 0.1)
    in fp32 (a trained norm weight stays near its initial value of 1)."""
    gen = torch.Generator(device=draw_device or "cpu").manual_seed(seed)
    dd = draw_device or "cpu"
    gate = torch.randn(T, H, d_v, generator=gen, device=dd).to(dtype)
    weight = 1.0 + 0.1 * torch.randn(d_v, generator=gen, device=dd)
    return {"gate_raw": gate.to(device), "norm_weight": weight.to(device)}
