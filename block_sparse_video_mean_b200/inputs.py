"""Seeded synthetic Q/K/V for the block-sparse video attention forward.

This module only draws random numbers; it holds none of the attention method's
arithmetic, so both the CUDA path and the fp64 oracle may take their inputs from it.

Recipe (one generator per (batch b, head h), seeded with ``head_seed``):

* the rows of a head are split into groups: every run of ``block`` consecutive video
  rows is one group (a ragged tail run is a group of its own) and all sink rows form
  one more group;
* for each tensor X in (Q, K, V), in that order: draw the group vectors
  ``c_X ~ N(0, 1)^(groups x d)`` and then the noise ``eps_X ~ N(0, 1)^(N x d)``;
* ``X[t] = amp * c_X[group(t)] + eps_X[t]`` in fp32, rounded to bf16 (nearest even).

The block-shared component makes mean-pooled block scores informative, the way
neighbouring video tokens are correlated in a video-diffusion transformer; with
``amp = 0.5`` it carries 20% of the per-element variance.

``q_offset > 0`` adds one more draw per head, after the six above (so the other tensors
are unchanged): an offset vector ``o ~ N(0, 1)^d`` added to every query row as
``q_offset * o``. Real attention heads have a strong mean query direction; without it
the mean query (the compressed branch's anchor) is short and every anchor score of a
block is nearly equal. With ``q_offset = 1`` at d = 128 the anchor scores of a block
spread by about one unit, so the block's log-mass bias departs from log 64 by O(1).

On ``device="cpu"`` the draw uses torch's CPU generator; on a CUDA device it uses
torch's CUDA generator (a different stream of numbers). Either way, whichever side
compares against the oracle copies the very same tensors to the host.
"""
from __future__ import annotations

import torch

BLOCK = 64


def head_seed(seed: int, b: int, h: int, H: int) -> int:
    """Seed of the generator of head (b, h)."""
    return int(seed) * 1_000_003 + b * H + h


def _groups(n_video: int, n_sink: int, block: int) -> torch.Tensor:
    nvb = (n_video + block - 1) // block
    g = torch.arange(n_video) // block
    s = torch.full((n_sink,), nvb, dtype=torch.long)
    return torch.cat([g, s]), nvb + (1 if n_sink > 0 else 0)


def make_qkv(B: int, H: int, n_video: int, n_sink: int, d: int, seed: int = 0,
             device: str | torch.device = "cpu", block: int = BLOCK, amp: float = 0.5,
             q_offset: float = 0.0):
    """Return (Q, K, V), each bf16 [B, H, n_video + n_sink, d] on ``device``."""
    device = torch.device(device)
    N = n_video + n_sink
    group, ngroups = _groups(n_video, n_sink, block)
    group = group.to(device)
    out = [torch.empty((B, H, N, d), dtype=torch.bfloat16, device=device) for _ in range(3)]
    for b in range(B):
        for h in range(H):
            g = torch.Generator(device=device)
            g.manual_seed(head_seed(seed, b, h, H))
            xs = []
            for X in out:
                c = torch.randn((max(ngroups, 1), d), generator=g, device=device, dtype=torch.float32)
                eps = torch.randn((N, d), generator=g, device=device, dtype=torch.float32)
                xs.append(amp * c[group] + eps if N else None)
            if q_offset > 0:
                o = torch.randn((d,), generator=g, device=device, dtype=torch.float32)
                if N:
                    xs[0] = xs[0] + q_offset * o
            if N:
                for X, x in zip(out, xs):
                    X[b, h] = x.to(torch.bfloat16)
    return tuple(out)


def random_orthogonal(d: int, seed: int) -> torch.Tensor:
    """A seeded random orthogonal d x d matrix (fp64, CPU), for invariance tests."""
    g = torch.Generator().manual_seed(seed)
    a = torch.randn((d, d), generator=g, dtype=torch.float64)
    qm, r = torch.linalg.qr(a)
    return qm * torch.sign(torch.diagonal(r))[None, :]
