"""Seeded synthetic inputs for the sparse global attention (no method arithmetic lives here).

These generators feed both the CUDA library and the CPU oracle with identical tensors. The value
recipe follows the multi-view workloads the Speed3R pages describe (VGGT / pi3 token geometry:
N views x P patch tokens per view, flattened view-major), with a shared direction planted into a
few key blocks so that block selection is not a coin toss:

  Q, K, V  = bf16(randn(L, H, d) / sqrt(d))
  u        = randn(d), normalised to unit length (one per layer, shared by every head)
  boosted  = the first round(boost_frac * nb) entries of randperm(nb): those key blocks get
             K += boost * u on every token and head, before the bf16 cast
  gates    = randn(L, H, 2) fp32  (channel 0: compression gate logit, 1: selection gate logit)

Draw order on one torch Generator seeded with ``seed``: Q, K, V, u, the block permutation, gates.
``planted`` adds a second, optional stress distribution in which most query blocks have a clearly
separated top-k (graded boosts along per-group directions); see ``make_planted``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass
class Inputs:
    q: torch.Tensor      # [L, H, d] bf16
    k: torch.Tensor      # [L, H, d] bf16
    v: torch.Tensor      # [L, H, d] bf16
    gates: torch.Tensor  # [L, H, 2] fp32
    boosted: torch.Tensor  # indices of the boosted key blocks (int64)


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _randn_bf16(shape, g, device, d, chunk_rows: int = 1 << 18) -> torch.Tensor:
    """bf16(randn / sqrt(d)) drawn in row chunks so that huge tensors need no fp32 copy."""
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    inv = 1.0 / math.sqrt(d)
    for r0 in range(0, shape[0], chunk_rows):
        r1 = min(shape[0], r0 + chunk_rows)
        x = torch.randn((r1 - r0,) + tuple(shape[1:]), generator=g, device=device,
                        dtype=torch.float32)
        out[r0:r1] = (x * inv).to(torch.bfloat16)
    return out


def make_inputs(L: int, H: int, d: int, block: int, seed: int, device="cpu",
                boost_frac: float = 0.05, boost: float = 3.0) -> Inputs:
    """The standard workload distribution (see module docstring)."""
    g = _gen(device, seed)
    q = _randn_bf16((L, H, d), g, device, d)
    # K stays fp32 until the boost (drawn after V) has been added, then is cast once
    k32 = torch.randn((L, H, d), generator=g, device=device, dtype=torch.float32)
    k32 *= 1.0 / math.sqrt(d)
    v = _randn_bf16((L, H, d), g, device, d)
    u = torch.randn(d, generator=g, device=device, dtype=torch.float32)
    u = u / u.norm()
    nb = -(-L // block)
    nboost = int(round(boost_frac * nb))
    perm = torch.randperm(nb, generator=g, device=device)
    boosted = perm[:nboost].sort().values
    for j in boosted.tolist():
        k32[j * block:min(L, (j + 1) * block)] += boost * u
    k = k32.to(torch.bfloat16)
    del k32
    gates = torch.randn((L, H, 2), generator=g, device=device, dtype=torch.float32)
    return Inputs(q, k, v, gates, boosted)


def make_planted(L: int, H: int, d: int, block: int, seed: int, device="cpu", groups: int = 4,
                 qboost: float = 1.0) -> Inputs:
    """Stress distribution with well-separated top-k sets.

    Query block i belongs to group i % groups and key block j to group j % groups; each group has
    its own random unit direction w_g. Every query of a group-g block gets Q += qboost * w_g, and
    every token of key block j gets K += c_j * w_{g(j)} with c_j graded in [0.5, 3] by a seeded
    permutation, so a query block ranks the key blocks of its own group by their grade.
    """
    g = _gen(device, seed)
    qblock = 64
    q32 = torch.randn((L, H, d), generator=g, device=device) / math.sqrt(d)
    k32 = torch.randn((L, H, d), generator=g, device=device) / math.sqrt(d)
    v = _randn_bf16((L, H, d), g, device, d)
    w = torch.randn((groups, d), generator=g, device=device)
    w = w / w.norm(dim=1, keepdim=True)
    nb = -(-L // block)
    grade = torch.randperm(nb, generator=g, device=device).to(torch.float32)
    grade = 0.5 + 2.5 * grade / max(1, nb - 1)
    tok = torch.arange(L, device=device)
    q32 += qboost * w[(tok // qblock) % groups][:, None, :]
    kb = tok // block
    k32 += (grade[kb][:, None] * w[kb % groups])[:, None, :]
    gates = torch.randn((L, H, 2), generator=g, device=device, dtype=torch.float32)
    return Inputs(q32.to(torch.bfloat16), k32.to(torch.bfloat16), v, gates,
                  torch.zeros(0, dtype=torch.int64, device=device))
