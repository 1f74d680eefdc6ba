"""Seeded synthetic inputs for the MoE layer (shared by the CUDA path's tests and bench
and by the oracle's tests).

This module holds the input recipe only, none of the layer's arithmetic:

* x = z / sqrt(mean(z^2) + 1e-6) per token, z ~ N(0, 1), then cast to the config dtype
  (the layer's input is the RMS-normalised stream, "GLM-4.5 MoE Forward", How it
  works; the normaliser has no gain and eps 1e-6 here).
* W_g, gate_up_proj, down_proj and the shared expert's matrices ~ N(0, 0.02^2).
* correction bias b ~ U(-beta, beta), fp32.
* skewed configurations add to router row pi(r) the offset a (r+1)^(-gamma) u_pi(r),
  where pi is a seeded permutation of the experts, r the popularity rank and u_e a
  seeded unit vector per expert.  With zero-mean x this raises the logit variance of
  low-rank experts, so they win the top-k more often.  gamma is the Zipf exponent
  1.1 and `a` was bisected (oracle/fit_skew.py) so that the load of a calibration
  batch has max/mean 10 (its popularity-rank log-log slope comes out near -1.45;
  top-8-of-256 selection saturates the head, so no (a, gamma) reaches slope -1.1
  together with 10x max/mean).

Weights are generated one expert at a time so that fp32 temporaries stay small.
"""

from __future__ import annotations

import dataclasses

import torch

from .configs import MoEConfig

# Fitted by oracle/fit_skew.py (see its docstring); recorded here as constants.
SKEW_A = 11.0993
SKEW_GAMMA = 1.1
SKEW_SEED_OFFSET = 7919


@dataclasses.dataclass
class MoEInputs:
    x: torch.Tensor  # [N, D]
    W_g: torch.Tensor  # [E, D]
    b: torch.Tensor  # [E] fp32
    gate_up: torch.Tensor  # [E, 2 d_moe, D]; rows 0..d-1 gate, d..2d-1 up
    down: torch.Tensor  # [E, D, d_moe]
    sh_gate: torch.Tensor  # [d_sh, D]
    sh_up: torch.Tensor  # [d_sh, D]
    sh_down: torch.Tensor  # [D, d_sh]

    def to(self, device) -> "MoEInputs":
        return MoEInputs(**{f.name: getattr(self, f.name).to(device)
                            for f in dataclasses.fields(self)})


def _normal(shape, g, device, std=0.02):
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std


def rms_normalised_tokens(N: int, D: int, g: torch.Generator, device) -> torch.Tensor:
    z = torch.randn((N, D), generator=g, device=device, dtype=torch.float32)
    return z * torch.rsqrt(z.pow(2).mean(dim=-1, keepdim=True) + 1e-6)


def skew_offsets(E: int, D: int, seed: int, device, a: float = SKEW_A,
                 gamma: float = SKEW_GAMMA) -> torch.Tensor:
    """Router-row offsets [E, D] giving Zipf-like expert popularity (see module doc)."""
    g = torch.Generator(device=device)
    g.manual_seed(seed + SKEW_SEED_OFFSET)
    perm = torch.randperm(E, generator=g, device=device)
    u = torch.randn((E, D), generator=g, device=device, dtype=torch.float32)
    u = u / u.norm(dim=1, keepdim=True)
    ranks = torch.arange(E, device=device, dtype=torch.float32)
    scale = a * (ranks + 1.0).pow(-gamma)
    off = torch.zeros((E, D), device=device, dtype=torch.float32)
    off[perm] = scale[:, None] * u[perm]
    return off


def router_inputs(cfg: MoEConfig, seed: int = 0, device="cpu"):
    """(x, W_g in fp32 before the dtype cast, b, generator) drawn exactly as make_inputs does."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    x = rms_normalised_tokens(cfg.N, cfg.D, g, device).to(cfg.dtype)
    wg = _normal((cfg.E, cfg.D), g, device)
    if cfg.skew:
        wg = wg + skew_offsets(cfg.E, cfg.D, seed, device)
    b = (torch.rand((cfg.E,), generator=g, device=device, dtype=torch.float32) * 2.0 - 1.0) * cfg.beta
    return x, wg, b, g


def make_inputs(cfg: MoEConfig, seed: int = 0, device="cpu") -> MoEInputs:
    """All layer inputs for `cfg`, generated with a torch generator on `device`."""
    x, wg, b, g = router_inputs(cfg, seed, device)
    W_g = wg.to(cfg.wg_dtype)
    E, D, d, dsh = cfg.E, cfg.D, cfg.d_moe, cfg.d_sh
    gate_up = torch.empty((E, 2 * d, D), dtype=cfg.dtype, device=device)
    down = torch.empty((E, D, d), dtype=cfg.dtype, device=device)
    for e in range(E):
        gate_up[e] = _normal((2 * d, D), g, device).to(cfg.dtype)
        down[e] = _normal((D, d), g, device).to(cfg.dtype)
    sh_gate = _normal((dsh, D), g, device).to(cfg.dtype)
    sh_up = _normal((dsh, D), g, device).to(cfg.dtype)
    sh_down = _normal((D, dsh), g, device).to(cfg.dtype)
    return MoEInputs(x, W_g, b, gate_up, down, sh_gate, sh_up, sh_down)


def make_tokens(cfg: MoEConfig, N: int, seed: int, device="cpu") -> torch.Tensor:
    """A fresh batch of N RMS-normalised tokens for cfg (used for calibration batches)."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return rms_normalised_tokens(N, cfg.D, g, device).to(cfg.dtype)
