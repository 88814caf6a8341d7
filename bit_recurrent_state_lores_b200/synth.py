"""Seeded synthetic decode workloads shaped like the LoReS pages' settings.

This module only draws inputs.  It holds none of the decode step's arithmetic,
so the CUDA path and the CPU oracle can both be fed from it.

Every workload produces, per decode step t, fp32 tensors
  q, k  [B, H, d_k]  unit L2 norm (the recurrence's domain constraint)
  v     [B, H, d_v]
  alpha [B, H] (scalar decay per head) or [B, H, d_k] (decay per key column)
  beta  [B, H]
drawn from a torch generator seeded by (seed, t), on any device.  Per-head
constants (decay time constants, decay means, outlier channels) are drawn once
from the seed on the CPU.

Recipes (the reading of each setting is stated beside it):
  tiny   batch 1, 2 heads, d_k = d_v = 16, 32 steps, delta rule, scalar decay
         alpha = exp(-softplus(x)), x ~ N(0,1) per step, beta = sigmoid(N(0,1)),
         int8 with one scale per value row, zero initial state, seed 0.
  gdn    batch 64, 32 heads, 128 x 128, 256 steps after a 64-step fp32 warmup,
         delta rule, alpha_h = exp(-1/tau_h) with tau_h log-uniform in [1, 1000]
         (tau read as an e-folding time), beta = sigmoid(N(0,1)), v ~ N(0,1) with
         4 value channels per head multiplied by 8, int8, one scale per 32 keys.
  mamba2 delta off, batch 128, 128 heads, d_v 64 x d_k 128, 512 steps,
         tau_h log-uniform in [1, 4096], beta = softplus(N(0,1)) clipped into
         [1e-6, 2 - 1e-6], int8 with one scale per value row.
  kda    batch 256, 32 heads, 128 x 128, 1024 steps, delta rule, decay per key
         column alpha = exp(-softplus(N(mu_h, 1))), mu_h chosen so the head mean
         decay runs from 0.5 to 0.9999 (1 - mean log-spaced 0.5 .. 1e-4, solved by
         bisection with 64-point Gauss-Hermite quadrature), 4 heavy value
         channels x8, the 25% slowest-decaying heads int8 and the rest int4.
  sweep  the gdn generators with one scale per value row, H = 32, 128 x 128,
         48 layers (each layer its own seed), batch in {1, 16, 64, 256, 1024}.
"""
from dataclasses import dataclass, field, replace
from typing import Optional

import numpy as np
import torch


@dataclass
class Workload:
    name: str
    B: int
    H: int
    d_k: int
    d_v: int
    steps: int
    delta: int = 1
    diag: int = 0
    group: Optional[int] = None          # None -> d_k (one scale per value row)
    bits: int = 8                        # uniform bits when mixed_frac is None
    mixed_frac: Optional[float] = None   # fraction of heads kept at 8 bits
    warmup: int = 0                      # fp32 warmup steps before quantizing
    decay: str = "tau"                   # "softplus_normal" | "tau" | "kda" | "kda_channel"
    tau_max: float = 1000.0
    beta_kind: str = "sigmoid"           # "sigmoid" | "softplus_clip"
    outliers: int = 0                    # value channels per head scaled x8
    seed: int = 0
    layers: int = 1
    extra: dict = field(default_factory=dict)

    @property
    def G(self):
        return self.group if self.group else self.d_k


WORKLOADS = {
    "tiny": Workload("tiny", B=1, H=2, d_k=16, d_v=16, steps=32, decay="softplus_normal",
                     seed=0),
    "gdn": Workload("gdn", B=64, H=32, d_k=128, d_v=128, steps=256, warmup=64, group=32,
                    decay="tau", tau_max=1000.0, outliers=4, seed=2),
    "mamba2": Workload("mamba2", B=128, H=128, d_k=128, d_v=64, steps=512, delta=0,
                       decay="tau", tau_max=4096.0, beta_kind="softplus_clip", seed=3),
    "kda": Workload("kda", B=256, H=32, d_k=128, d_v=128, steps=1024, diag=1, decay="kda",
                    mixed_frac=0.25, outliers=4, seed=4),
    "sweep": Workload("sweep", B=256, H=32, d_k=128, d_v=128, steps=128, warmup=16,
                      decay="tau", tau_max=1000.0, outliers=4, layers=48, seed=5),
}


def workload(name, **over):
    return replace(WORKLOADS[name], **over)


def _solve_mu(targets):
    """mu with E[exp(-softplus(mu + Z))] = m for each target m (Z ~ N(0, 1)): 64-point
    Gauss-Hermite quadrature and bisection, elementwise over an array of targets."""
    z, w = np.polynomial.hermite.hermgauss(64)
    z = z * np.sqrt(2.0)
    w = w / np.sqrt(np.pi)
    targets = np.asarray(targets, np.float64)
    lo = np.full(targets.shape, -40.0)
    hi = np.full(targets.shape, 40.0)             # the mean decay falls as mu rises
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        md = np.sum(w / (1.0 + np.exp(mid[..., None] + z)), axis=-1)
        up = md > targets
        lo = np.where(up, mid, lo)
        hi = np.where(up, hi, mid)
    return 0.5 * (lo + hi)


def _kda_mu(H):
    """mu_h with E[exp(-softplus(mu_h + Z))] = m_h, 1 - m_h log-spaced 0.5 .. 1e-4."""
    targets = 1.0 - np.logspace(np.log10(0.5), np.log10(1e-4), H)
    return _solve_mu(targets), targets


def _kda_channel_mu(H, d_k, g):
    """Per-channel decay means: in every head the d_k key channels span 1 - m log-spaced
    0.5 .. 1e-4 in a seeded random order, so the slow channels of a head are scattered
    over its key groups."""
    base = 1.0 - np.logspace(np.log10(0.5), np.log10(1e-4), d_k)
    targets = np.stack([base[torch.randperm(d_k, generator=g).numpy()] for _ in range(H)])
    return _solve_mu(targets), targets


def head_params(wl: Workload, layer: int = 0):
    """Per-head constants: dict with 'alpha_h' (scalar decay, or None),
    'mu' (kda), 'mean_decay' [H], 'outlier_idx' [H, outliers]."""
    g = torch.Generator().manual_seed(wl.seed * 7919 + layer * 104729 + 17)
    out = {"alpha_h": None, "mu": None}
    if wl.decay == "tau":
        u = torch.rand(wl.H, generator=g, dtype=torch.float64)
        tau = torch.exp(u * np.log(wl.tau_max))          # log-uniform in [1, tau_max]
        alpha_h = torch.exp(-1.0 / tau).to(torch.float32)
        out["alpha_h"] = alpha_h
        out["mean_decay"] = alpha_h.numpy().astype(np.float32)
    elif wl.decay == "kda":
        mu, target = _kda_mu(wl.H)
        out["mu"] = torch.tensor(mu, dtype=torch.float32)
        out["mean_decay"] = target.astype(np.float32)
    elif wl.decay == "kda_channel":
        mu, target = _kda_channel_mu(wl.H, wl.d_k, g)
        out["mu"] = torch.tensor(mu, dtype=torch.float32)                  # [H, d_k]
        out["mean_decay_channel"] = target.astype(np.float32)              # [H, d_k]
        out["mean_decay"] = target.mean(axis=1).astype(np.float32)
    else:  # softplus_normal: E[exp(-softplus(Z))] = E[sigmoid(-Z)] = 1/2 for every head
        out["mean_decay"] = np.full(wl.H, 0.5, np.float32)
    if wl.outliers:
        idx = torch.stack([torch.randperm(wl.d_v, generator=g)[:wl.outliers] for _ in range(wl.H)])
        out["outlier_idx"] = idx
    else:
        out["outlier_idx"] = None
    return out


def head_bits(wl: Workload, hp=None):
    """Bits per head.  Mixed precision goes through the library's own policy
    helper at create time; this returns the uniform case only."""
    if wl.mixed_frac is None:
        return [wl.bits] * wl.H
    return None


def _unit(x):
    return x / torch.linalg.vector_norm(x, dim=-1, keepdim=True)


def step_inputs(wl: Workload, step: int, hp=None, device="cpu", layer: int = 0, B=None):
    """(q, k, v, alpha, beta) for decode step `step`, contiguous fp32 on `device`."""
    if hp is None:
        hp = head_params(wl, layer)
    B = wl.B if B is None else B
    H, dk, dv = wl.H, wl.d_k, wl.d_v
    g = torch.Generator(device=device).manual_seed(
        (wl.seed * 1000003 + layer * 8191 + step * 131071 + 1) & 0x7FFFFFFFFFFFFFFF)
    kw = dict(generator=g, device=device, dtype=torch.float32)
    q = _unit(torch.randn(B, H, dk, **kw))
    k = _unit(torch.randn(B, H, dk, **kw))
    v = torch.randn(B, H, dv, **kw)
    if hp["outlier_idx"] is not None:
        scale = torch.ones(H, dv, dtype=torch.float32)
        scale.scatter_(1, hp["outlier_idx"], 8.0)
        v = v * scale.to(device)[None]
    if wl.beta_kind == "sigmoid":
        beta = torch.sigmoid(torch.randn(B, H, **kw))
    else:
        beta = torch.nn.functional.softplus(torch.randn(B, H, **kw)).clamp(1e-6, 2.0 - 1e-6)
    if wl.decay == "softplus_normal":
        alpha = torch.exp(-torch.nn.functional.softplus(torch.randn(B, H, **kw)))
    elif wl.decay == "tau":
        alpha = hp["alpha_h"].to(device)[None].expand(B, H).contiguous()
    else:
        mu = hp["mu"].to(device)
        y = torch.randn(B, H, dk, **kw) + (mu[None, :, None] if mu.dim() == 1 else mu[None])
        alpha = torch.exp(-torch.nn.functional.softplus(y))
    return (q.contiguous(), k.contiguous(), v.contiguous(), alpha.contiguous(),
            beta.contiguous())
