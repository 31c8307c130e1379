"""Seeded synthetic inputs for the gated delta-rule path.

This module is shared by the CUDA path's tests and benchmark and by the
oracle's tests.  It holds only the input recipe (random draws, the
normalisation and gate parameterisation that define the workloads); none of
the method's own arithmetic (decay, readout, erase/write, the Kaczmarz step)
is here.

Recipe (fixed draw order from one ``torch.Generator`` seeded with ``seed``,
all draws fp32 on the CPU):

1. q ~ N(0,1) [B,T,H,dk];  k ~ N(0,1) [B,T,H,dk];  v ~ N(0,1) [B,T,H,dv]
2. beta_logit ~ N(0,1) [B,T,H]
3. decay_logit ~ N(0,1): [B,T,H] for scalar-decay variants and DeltaNet,
   [B,T,H,dk] for channel-wise decay (KDA, GDN-2)
4. GDN-2 only: erase_logit, write_logit ~ N(0,1) [B,T,H,dk]
5. KLA only: key_scale = exp(0.5 * N(0,1)) [B,T,H]  (LogNormal(0, 0.5))

Then: q is L2-normalised per (token, head); k is L2-normalised except for KLA,
whose keys are k / sqrt(dk) * key_scale (unnormalised, N(0, 1/dk) scaled per
token); beta = sigmoid(beta_logit) (eta for KLA); log_g = -softplus(decay_logit)
so that g = exp(log_g) = sigmoid(-decay_logit) lies in (0, 1); GDN-2 gates are
sigmoid of their logits, or, with ``gdn2_tied``, both equal to beta broadcast
over dk.  q, k, v are cast to the I/O dtype last; the gates stay fp32.

DeltaNet draws the same tensors as Gated DeltaNet and ignores the decay, so
both run on identical q, k, v, beta for the same seed; KDA and tied GDN-2 draw
identical q, k, v, beta and log_g for the same seed.
"""
from __future__ import annotations

import torch
import torch.nn.functional as F

VARIANT_NAMES = ("deltanet", "gdn", "kda", "gdn2", "kla")
CHANNEL_DECAY = ("kda", "gdn2")


def _l2n(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-6)


def make_inputs(variant: str, B: int, T: int, H: int, dk: int = 128, dv: int = 128,
                dtype: torch.dtype = torch.bfloat16, seed: int = 0,
                gdn2_tied: bool = False) -> dict:
    """CPU tensors {q,k,v,beta,log_g,erase_b,write_w}; unused gates are None."""
    if variant not in VARIANT_NAMES:
        raise ValueError(f"unknown variant {variant!r}")
    g = torch.Generator().manual_seed(int(seed))
    q = torch.randn(B, T, H, dk, generator=g)
    k = torch.randn(B, T, H, dk, generator=g)
    v = torch.randn(B, T, H, dv, generator=g)
    beta_logit = torch.randn(B, T, H, generator=g)
    channel = variant in CHANNEL_DECAY
    decay_logit = torch.randn(*((B, T, H, dk) if channel else (B, T, H)), generator=g)
    erase_b = write_w = None
    if variant == "gdn2":
        erase_logit = torch.randn(B, T, H, dk, generator=g)
        write_logit = torch.randn(B, T, H, dk, generator=g)
    if variant == "kla":
        key_scale = torch.exp(0.5 * torch.randn(B, T, H, generator=g))
        k = k / (dk ** 0.5) * key_scale[..., None]
    else:
        k = _l2n(k)
    q = _l2n(q)
    beta = torch.sigmoid(beta_logit)
    log_g = None if variant == "deltanet" else -F.softplus(decay_logit)
    if variant == "gdn2":
        if gdn2_tied:
            erase_b = beta[..., None].expand(B, T, H, dk).contiguous()
            write_w = erase_b.clone()
        else:
            erase_b = torch.sigmoid(erase_logit)
            write_w = torch.sigmoid(write_logit)
        beta = None
    return {
        "q": q.to(dtype).contiguous(), "k": k.to(dtype).contiguous(),
        "v": v.to(dtype).contiguous(), "beta": beta, "log_g": log_g,
        "erase_b": erase_b, "write_w": write_w,
    }


def make_raw_inputs(variant: str, B: int, T: int, H: int, dk: int = 128, dv: int = 128,
                    dtype: torch.dtype = torch.bfloat16, seed: int = 0) -> dict:
    """The same draws as make_inputs, before the transforms: q and k as drawn
    (KLA's k already scaled by 1/sqrt(dk) and the key scale, since that is its
    key), v, and the logits of beta (eta), of the decay and of the GDN-2 gates.
    q, k, v in the I/O dtype, the logits fp32.  For the raw-input mode."""
    if variant not in VARIANT_NAMES:
        raise ValueError(f"unknown variant {variant!r}")
    g = torch.Generator().manual_seed(int(seed))
    q = torch.randn(B, T, H, dk, generator=g)
    k = torch.randn(B, T, H, dk, generator=g)
    v = torch.randn(B, T, H, dv, generator=g)
    beta_logit = torch.randn(B, T, H, generator=g)
    channel = variant in CHANNEL_DECAY
    decay_logit = torch.randn(*((B, T, H, dk) if channel else (B, T, H)), generator=g)
    erase_logit = write_logit = None
    if variant == "gdn2":
        erase_logit = torch.randn(B, T, H, dk, generator=g)
        write_logit = torch.randn(B, T, H, dk, generator=g)
    if variant == "kla":
        key_scale = torch.exp(0.5 * torch.randn(B, T, H, generator=g))
        k = k / (dk ** 0.5) * key_scale[..., None]
    return {
        "q": q.to(dtype).contiguous(), "k": k.to(dtype).contiguous(), "v": v.to(dtype).contiguous(),
        "beta": None if variant == "gdn2" else beta_logit.contiguous(),
        "log_g": None if variant == "deltanet" else decay_logit.contiguous(),
        "erase_b": None if erase_logit is None else erase_logit.contiguous(),
        "write_w": None if write_logit is None else write_logit.contiguous(),
    }


def transform_raw(variant: str, raw: dict) -> dict:
    """The input transforms applied to raw inputs, in float64 on the exact
    values passed (the I/O-dtype q, k, v up-cast): unit q, unit k except KLA's,
    sigmoid of beta / eta and of the GDN-2 gates, log_g = -softplus.  What the
    raw-input mode of the kernels is compared against."""
    f = lambda x: None if x is None else x.double()
    q, k = f(raw["q"]), f(raw["k"])
    q = q / q.norm(dim=-1, keepdim=True).clamp_min(1e-6)
    if variant != "kla":
        k = k / k.norm(dim=-1, keepdim=True).clamp_min(1e-6)
    sig = lambda x: None if x is None else torch.sigmoid(x.double())
    return {
        "q": q, "k": k, "v": f(raw["v"]), "beta": sig(raw["beta"]),
        "log_g": None if raw["log_g"] is None else -F.softplus(raw["log_g"].double()),
        "erase_b": sig(raw["erase_b"]), "write_w": sig(raw["write_w"]),
    }


def make_decode_inputs(variant: str, N: int, H: int, step: int, dk: int = 128, dv: int = 128,
                       dtype: torch.dtype = torch.bfloat16, base_seed: int = 1000) -> dict:
    """Inputs of decode step ``step`` for N sequences (seed base_seed + step); [N,H,...]."""
    d = make_inputs(variant, N, 1, H, dk, dv, dtype, seed=base_seed + step)
    return {name: (None if t is None else t[:, 0].contiguous()) for name, t in d.items()}


def random_state(B: int, H: int, dk: int, dv: int, seed: int, scale: float = 0.5) -> torch.Tensor:
    """A seeded fp32 state [B,H,dk,dv] (for initial-state and decode tests)."""
    g = torch.Generator().manual_seed(int(seed))
    return (scale * torch.randn(B, H, dk, dv, generator=g)).contiguous()


def random_output_grad(B: int, T: int, H: int, dv: int, seed: int, dtype: torch.dtype = torch.bfloat16,
                       scale: float = 1.0) -> torch.Tensor:
    """A seeded gradient of the outputs d_o [B,T,H,dv] ~ scale * N(0, 1) (for the backward)."""
    g = torch.Generator().manual_seed(int(seed))
    return (scale * torch.randn(B, T, H, dv, generator=g)).to(dtype).contiguous()
