"""Seeded synthetic inputs for causal linear attention.

This module draws the inputs of the standard workloads and nothing else: it
holds none of the method's arithmetic, so the CUDA path and the float64 oracle
can both be fed from it without sharing any computation.

Recipe (every workload): a ``torch.Generator`` seeded with ``seed`` (0 by
default) on the chosen device draws q, then k, then v as float32 standard
normals of shape [B, T, H, d]; each is multiplied by ``scale`` and cast to the
workload dtype.  Packed variable-length batches first draw their lengths on a
CPU generator seeded the same way (``randint(lo, hi + 1, (n,))``), so the
lengths do not depend on the device.  Decode workloads draw q, k, v of shape
[N, H, d] and then the state [N, H, d_k, d_v] as ``state_std`` * N(0, 1).
Workloads with a data-dependent decay then draw its log, g [B, T, H], uniform
in [ln lo, ln hi] (``gate = (lo, hi)``), from a second generator seeded with seed + 1,
and gated-delta workloads a write strength beta [B, T, H] uniform in [0.1, 1) after it.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    H: int
    d_k: int
    d_v: int
    dtype: str  # "f32" or "bf16"
    scale: float
    gamma: tuple  # per-head decay, len H
    phi: str  # "identity" or "elu1"
    normalize: bool
    chunk: int = 64
    varlen: Optional[tuple] = None  # (n_seqs, lo, hi) for packed batches
    gate: Optional[tuple] = None  # (lo, hi): per-token decays in [lo, hi] (log drawn uniform)
    delta: bool = False  # gated delta rule: also a write strength beta per token, U[0.1, 1)
    gamma_rule: str = ""  # how the per-head decays were chosen (a label for reports)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


def retnet_gammas(H: int, shift: int) -> tuple:
    """gamma_h = 1 - 2^(-shift-h), h = 0..H-1 (exact in float32 for these sizes)."""
    return tuple(1.0 - 2.0 ** (-shift - h) for h in range(H))


def linspace_gammas(H: int, lo: float, hi: float) -> tuple:
    """H decays evenly spaced in [lo, hi], as float32 values."""
    return tuple(float(x) for x in torch.linspace(lo, hi, H, dtype=torch.float32))


def _sweep(T: int) -> Workload:
    return Workload(
        f"sweep_B8_H16_d128_T{T}", B=8, T=T, H=16, d_k=128, d_v=128, dtype="bf16",
        scale=1.0 / math.sqrt(128), gamma=linspace_gammas(16, 0.9, 0.999),
        phi="identity", normalize=False, gamma_rule="evenly spaced in [0.9, 0.999]",
    )


WORKLOADS = {
    "tiny_f32": Workload(
        "tiny_f32_B1_H2_T256_d64", B=1, T=256, H=2, d_k=64, d_v=64, dtype="f32", scale=1.0,
        gamma=(1.0, 1.0), phi="elu1", normalize=True, gamma_rule="1 (no decay)",
    ),
    "retnet_d256": Workload(
        "retnet_B32_H4_T2048_d256", B=32, T=2048, H=4, d_k=256, d_v=256, dtype="bf16",
        scale=1.0 / math.sqrt(256), gamma=retnet_gammas(4, 5), phi="identity", normalize=False,
        gamma_rule="1 - 2^(-5-h), h = 0..3",
    ),
    "sweep_T4096": _sweep(4096),
    "sweep_T8192": _sweep(8192),
    "sweep_T16384": _sweep(16384),
    "varlen": Workload(
        "varlen_64seqs_L128-2048_H8_d128", B=1, T=0, H=8, d_k=128, d_v=128, dtype="bf16",
        scale=1.0 / math.sqrt(128), gamma=(1.0,) * 8, phi="elu1", normalize=True,
        varlen=(64, 128, 2048), gamma_rule="1 (no decay)",
    ),
    "gated_T16384": Workload(
        "gated_B8_H16_d128_T16384", B=8, T=16384, H=16, d_k=128, d_v=128, dtype="bf16",
        scale=1.0 / math.sqrt(128), gamma=(1.0,) * 16, phi="identity", normalize=False, gate=(0.9, 0.999),
        gamma_rule="per token: exp(g), g uniform in [ln 0.9, ln 0.999]",
    ),
    "gdelta_T16384": Workload(
        "gated_delta_B8_H16_d128_T16384", B=8, T=16384, H=16, d_k=128, d_v=128, dtype="bf16",
        scale=1.0 / math.sqrt(128), gamma=(1.0,) * 16, phi="identity", normalize=False, gate=(0.9, 0.999),
        delta=True, gamma_rule="per token: exp(g), g uniform in [ln 0.9, ln 0.999]; beta uniform in [0.1, 1)",
    ),
    "long_1m": Workload(
        "long_B1_H4_T1048576_d128", B=1, T=1 << 20, H=4, d_k=128, d_v=128, dtype="bf16",
        scale=1.0 / math.sqrt(128), gamma=retnet_gammas(4, 8), phi="identity", normalize=False,
        gamma_rule="1 - 2^(-8-h), h = 0..3",
    ),
}

# Decode: N states of [d_k, d_v] (fp32), one token each.
DECODE = dict(name="decode_N256_H4_d128", N=256, H=4, d_k=128, d_v=128, state_std=0.01,
              scale=1.0 / math.sqrt(128), gamma=retnet_gammas(4, 8), phi="identity")


def varlen_lengths(n: int, lo: int, hi: int, seed: int = 0) -> torch.Tensor:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return torch.randint(lo, hi + 1, (n,), generator=g, dtype=torch.int64)


def cu_seqlens_from_lengths(lengths) -> torch.Tensor:
    lengths = torch.as_tensor(lengths, dtype=torch.int64)
    cu = torch.zeros(lengths.numel() + 1, dtype=torch.int64)
    cu[1:] = torch.cumsum(lengths, 0)
    return cu.to(torch.int32)


def make_qkv(B, T, H, d_k, d_v, dtype, scale, seed=0, device="cpu"):
    """Draw q, k, v ([B,T,H,d]) as described in the module docstring."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    out = []
    for d in (d_k, d_k, d_v):
        x = torch.randn((B, T, H, d), generator=g, device=device, dtype=torch.float32)
        if scale != 1.0:
            x.mul_(scale)
        out.append(x.to(dtype))
    return tuple(out)


def make_log_decay(B, T, H, lo, hi, generator, device="cpu"):
    """g [B, T, H] float32, uniform in [ln lo, ln hi] (decays exp(g) in [lo, hi])."""
    a, b = math.log(lo), math.log(hi)
    return torch.rand((B, T, H), generator=generator, device=device, dtype=torch.float32) * (b - a) + a


def make_inputs(w: Workload, seed: int = 0, device="cpu", T: Optional[int] = None, B: Optional[int] = None):
    """Inputs of workload ``w``: dict(q, k, v, gamma, cu_seqlens[, g]).

    ``T`` / ``B`` override the sequence length / batch (used to shrink a
    workload for a quick check while keeping its distribution).
    """
    cu = None
    if w.varlen is not None:
        n, lo, hi = w.varlen
        lengths = varlen_lengths(n, lo, hi, seed)
        cu = cu_seqlens_from_lengths(lengths)
        Bq, Tq = 1, int(cu[-1])
    else:
        Bq, Tq = (B if B is not None else w.B), (T if T is not None else w.T)
    q, k, v = make_qkv(Bq, Tq, w.H, w.d_k, w.d_v, w.torch_dtype, w.scale, seed, device)
    gamma = torch.tensor(w.gamma, dtype=torch.float32, device=device)
    if cu is not None:
        cu = cu.to(device)
    x = dict(q=q, k=k, v=v, gamma=gamma, cu_seqlens=cu)
    if w.gate is not None:
        gen = torch.Generator(device=device)
        gen.manual_seed(seed + 1)
        x["g"] = make_log_decay(Bq, Tq, w.H, w.gate[0], w.gate[1], gen, device)
        if w.delta:
            x["beta"] = torch.rand((Bq, Tq, w.H), generator=gen, device=device, dtype=torch.float32) * 0.9 + 0.1
    return x


def make_dout(v: torch.Tensor, seed: int = 0) -> torch.Tensor:
    """A seeded N(0, 1) output gradient shaped and typed like ``v`` (for the backward)."""
    g = torch.Generator(device=v.device)
    g.manual_seed(seed + 2)
    return torch.randn(v.shape, generator=g, device=v.device, dtype=torch.float32).to(v.dtype)


def make_norm_gate(v: torch.Tensor, seed: int = 0):
    """Gate (N(0, 1) * 2, like v) and norm weights (U[0.5, 1.5), [d_v]) for the output norm."""
    g = torch.Generator(device=v.device)
    g.manual_seed(seed + 3)
    gate = (torch.randn(v.shape, generator=g, device=v.device) * 2.0).to(v.dtype)
    w = torch.rand(v.shape[-1], generator=g, device=v.device) + 0.5
    return gate, w


def make_decode_inputs(N, H, d_k, d_v, scale, state_std, gamma, seed=0, device="cpu",
                       dtype=torch.float32):
    """Decode inputs: q, k [N,H,d_k], v [N,H,d_v], state [N,H,d_k,d_v] fp32, gamma [H]."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    q = (torch.randn((N, H, d_k), generator=g, device=device) * scale).to(dtype)
    k = (torch.randn((N, H, d_k), generator=g, device=device) * scale).to(dtype)
    v = (torch.randn((N, H, d_v), generator=g, device=device) * scale).to(dtype)
    state = torch.randn((N, H, d_k, d_v), generator=g, device=device) * state_std
    gam = torch.tensor(gamma, dtype=torch.float32, device=device)
    return dict(q=q, k=k, v=v, state=state, gamma=gam)
