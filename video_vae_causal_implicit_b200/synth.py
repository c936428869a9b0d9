"""Seeded synthetic inputs for the causal Conv3D and the residual block.

This module only draws random numbers; it holds none of the convolution,
normalisation or activation arithmetic.  Tests feed the same tensors to the
CUDA library and to the CPU oracle, and the benchmark uses it for its
synthetic workloads.

Recipe (the same for every workload):
  * a ``torch.Generator`` seeded per tensor, drawing in the logical
    [N, C, T, H, W] order the pages use;
  * activations ~ N(0, 1) (the encoder video input ~ U(-1, 1));
  * conv weights: Kaiming-uniform, bound sqrt(6 / fan_in),
    fan_in = C_in * kt * kh * kw;
  * conv bias ~ U(-0.1, 0.1); RMS gamma ~ U(0.5, 1.5);
  * bf16 tensors are rounded from the fp32 draw (round to nearest even),
    then permuted to channels-last NDHWC for the library.
Seeds: x 0, W1 1, b1 2, gamma1 3, W2 4, b2 5, gamma2 6 (plus ``seed_base``).
"""
from __future__ import annotations

import math

import torch

SEED_X, SEED_W1, SEED_B1, SEED_G1, SEED_W2, SEED_B2, SEED_G2 = range(7)


def _gen(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal(shape, seed, dtype=torch.bfloat16, device="cpu"):
    x = torch.randn(*shape, generator=_gen(seed, device), dtype=torch.float32, device=device)
    return x.to(dtype)


def uniform(shape, lo, hi, seed, dtype=torch.float32, device="cpu"):
    x = torch.empty(*shape, dtype=torch.float32, device=device)
    x.uniform_(lo, hi, generator=_gen(seed, device))
    return x.to(dtype)


def kaiming_uniform(cout, cin, k=(3, 3, 3), seed=1, dtype=torch.bfloat16):
    fan_in = cin * k[0] * k[1] * k[2]
    bound = math.sqrt(6.0 / fan_in)
    return uniform((cout, cin) + tuple(k), -bound, bound, seed, dtype)


def ndhwc(x_ncthw: torch.Tensor) -> torch.Tensor:
    """Contiguous channels-last copy [N, T, H, W, C] of a [N, C, T, H, W] tensor."""
    return x_ncthw.permute(0, 2, 3, 4, 1).contiguous()


def ncthw_view(x_ndhwc: torch.Tensor) -> torch.Tensor:
    """Logical [N, C, T, H, W] view of a channels-last tensor (no copy)."""
    return x_ndhwc.permute(0, 4, 1, 2, 3)


def conv_case(cin, cout, t, h, w, *, n=1, dtype=torch.bfloat16, seed_base=0,
              x_dist="normal", k=(3, 3, 3)):
    """One causal conv layer: x [N,Cin,T,H,W], W [Cout,Cin,k], bias [Cout] fp32."""
    if x_dist == "normal":
        x = normal((n, cin, t, h, w), seed_base + SEED_X, dtype)
    else:
        x = uniform((n, cin, t, h, w), -1.0, 1.0, seed_base + SEED_X, dtype)
    wt = kaiming_uniform(cout, cin, k, seed_base + SEED_W1, dtype)
    b = uniform((cout,), -0.1, 0.1, seed_base + SEED_B1, torch.float32)
    return {"x": x, "w": wt, "b": b}


def block_case(c, t, h, w, *, n=1, seed_base=0):
    """Residual block: x, (W1, b1, gamma1), (W2, b2, gamma2)."""
    x = normal((n, c, t, h, w), seed_base + SEED_X)
    return {
        "x": x,
        "w1": kaiming_uniform(c, c, (3, 3, 3), seed_base + SEED_W1),
        "b1": uniform((c,), -0.1, 0.1, seed_base + SEED_B1),
        "g1": uniform((c,), 0.5, 1.5, seed_base + SEED_G1),
        "w2": kaiming_uniform(c, c, (3, 3, 3), seed_base + SEED_W2),
        "b2": uniform((c,), -0.1, 0.1, seed_base + SEED_B2),
        "g2": uniform((c,), 0.5, 1.5, seed_base + SEED_G2),
    }


def sample_points(n, t, h, w, count, seed, frames=None):
    """Output voxels for sampled checks: every voxel of ``frames`` (if given)
    plus ``count`` seeded random voxels.  Rows are (n, t, h, w), int32."""
    rows = []
    if frames:
        for f in frames:
            if 0 <= f < t:
                hh, ww = torch.meshgrid(torch.arange(h), torch.arange(w), indexing="ij")
                for b in range(n):
                    rows.append(torch.stack([torch.full_like(hh, b), torch.full_like(hh, f),
                                             hh, ww], dim=-1).reshape(-1, 4))
    if count:
        g = _gen(seed)
        rows.append(torch.stack([torch.randint(0, n, (count,), generator=g),
                                 torch.randint(0, t, (count,), generator=g),
                                 torch.randint(0, h, (count,), generator=g),
                                 torch.randint(0, w, (count,), generator=g)], dim=-1))
    if not rows:
        return torch.zeros((0, 4), dtype=torch.int32)
    return torch.cat(rows).to(torch.int32)
