"""Seeded synthetic inputs for CLEAR attention (shared by the tests, the bench and the oracle checks).

This module draws random tensors and names workloads; it holds none of the attention arithmetic.
Every tensor is i.i.d. N(0, 1), drawn in float32 and then rounded to the requested dtype.
Draw order is fixed: q, k, v, then dO.

Workload shapes follow the FLUX attention calls described on the CLEAR pages
("CLEAR: Conv-Like Linearization Revs Pre-Trained Diffusion Transformers Up", the atlas summary
"Approach" and the pith review "Core claim"): 24 heads of head dim 128, 512 text tokens placed
before the H x W image tokens, radius r in {8, 16, 32}.
"""
from __future__ import annotations

from dataclasses import dataclass, asdict

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    heads: int
    n_text: int
    H: int
    W: int
    d: int
    r: int

    @property
    def N(self) -> int:
        return self.H * self.W

    @property
    def T(self) -> int:
        return self.n_text + self.H * self.W

    def as_dict(self) -> dict:
        return asdict(self)


# Named workloads: a tiny CPU-checkable case and the FLUX-shaped calls at 1024^2, 2048^2 and
# 8192^2 pixels (64x64, 128x128 and 512x512 token grids after 16x patchify), plus the
# distillation backward shape.
WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 16, 16, 16, 64, 4),
    "flux1024_r8": Workload("flux1024_r8", 1, 24, 512, 64, 64, 128, 8),
    "flux1024_r16": Workload("flux1024_r16", 1, 24, 512, 64, 64, 128, 16),
    "flux1024_r32": Workload("flux1024_r32", 1, 24, 512, 64, 64, 128, 32),
    "flux2048_r16": Workload("flux2048_r16", 1, 24, 512, 128, 128, 128, 16),
    "8k_r8": Workload("8k_r8", 1, 24, 512, 512, 512, 128, 8),
    "8k_r32": Workload("8k_r32", 1, 24, 512, 512, 512, 128, 32),
    "bwd_flux1024_r32": Workload("bwd_flux1024_r32", 2, 24, 512, 64, 64, 128, 32),
}


def make_inputs(wl: Workload, seed: int = 0, dtype=torch.bfloat16, device="cpu",
                with_grad_out: bool = False):
    """Return (q, k, v[, dO]) of shape [B, heads, T, d], i.i.d. N(0,1) from `seed`.

    On the CPU the draw uses torch.Generator('cpu'); on a CUDA device it uses a CUDA generator
    with the same seed (a different stream of numbers, still deterministic per seed). Values are
    drawn in float32 and rounded to `dtype`.
    """
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    shape = (wl.B, wl.heads, wl.T, wl.d)
    out = []
    for _ in range(4 if with_grad_out else 3):
        t = torch.randn(shape, generator=gen, dtype=torch.float32, device=dev)
        out.append(t.to(dtype) if dtype != torch.float32 else t)
    return tuple(out)


def make_random(shape, seed: int, dtype=torch.bfloat16, device="cpu"):
    """One i.i.d. N(0,1) tensor of `shape` from `seed` (float32 draw, then rounded)."""
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    t = torch.randn(shape, generator=gen, dtype=torch.float32, device=dev)
    return t.to(dtype) if dtype != torch.float32 else t


def quantize_e4m3(t: torch.Tensor):
    """Encode t [B, heads, T, d] as OCP FP8 E4M3 codes with one scale per (batch, head): the scale
    maps the head's largest magnitude to 448 (the format's largest finite value) and the codes are
    t / scale rounded to nearest-even by torch's float8_e4m3fn cast. Returns (codes uint8, scale
    float32 [B, heads]); decode(codes) * scale approximates t."""
    amax = t.detach().float().abs().amax(dim=(2, 3)).clamp_min(1e-12)
    scale = amax / 448.0
    codes = (t.float() / scale[:, :, None, None]).to(torch.float8_e4m3fn).view(torch.uint8)
    return codes, scale
