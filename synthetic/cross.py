"""Seeded synthetic inputs for AnnCA cross-attention (prompt pruning per frame).

FAST-AR summary, section 2.B "AnnCA": a frame only needs the prompt tokens that
describe what it shows; the pages give no prompt length, hash width or data. The
generator imitates that structure:

  * per head, C concept directions drawn from N(0, I_d) and rescaled to norm sqrt(d);
  * prompt: L tokens, token l describes concept l mod C; its key is the concept
    direction plus N(0, sigma^2 I_d), its value N(0, 1);
  * queries: every frame shows A of the C concepts (drawn per frame, the same for
    all heads); each of its P positions shows one of them uniformly, and its query
    is that concept's direction plus N(0, sigma^2 I_d), drawn afresh per call;
  * every draw is rounded to bf16 (round to nearest even).

The Wan-2.1-1.3B-shaped case uses L = 512 prompt tokens, the text length of that
model family's text encoder (outside knowledge: the pages give no prompt length).
Hyperplanes are N(0, 1) draws rounded to bf16, one set shared by all heads, from a
seed of their own.

Nothing here implements the method: it only draws numbers.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass

import torch

from .workload import round_to_bf16


@dataclass(frozen=True)
class CrossConfig:
    name: str
    H: int          # heads
    d: int          # head dimension
    P: int          # query tokens per frame
    F: int          # frames per query block
    L: int          # prompt tokens
    C: int          # concepts per head
    A: int          # concepts shown per frame
    sigma: float    # noise standard deviation of keys and queries
    nbits: int      # hash bits
    seed: int

    @property
    def T(self) -> int:
        return self.P * self.F

    def replace(self, **kw) -> "CrossConfig":
        return dataclasses.replace(self, **kw)


CROSS_CONFIGS = {
    "annca-tiny": CrossConfig("annca-tiny", 2, 64, 96, 3, 40, 8, 2, 0.15, 6, 2001),
    "annca-wan1.3b": CrossConfig("annca-wan1.3b", 12, 128, 1560, 3, 512, 32, 4, 0.25, 10, 2002),
}


def draw_cross_hyperplanes(nbits: int, d: int, seed: int) -> torch.Tensor:
    """N(0,1) normals rounded to bf16 values, [nbits, d] fp32 on the CPU."""
    g = torch.Generator(device="cpu").manual_seed(int(seed) * 104729 + 31)
    return round_to_bf16(torch.randn(nbits, d, generator=g, dtype=torch.float32))


class CrossWorkload:
    """prompt() -> (Kp, Vp) [L, H, d] bf16; queries(call) -> Q [F*P, H, d] bf16."""

    def __init__(self, cfg: CrossConfig, device="cpu"):
        self.cfg = cfg
        self.device = torch.device(device)
        g = torch.Generator(device=self.device).manual_seed(cfg.seed)
        concepts = torch.randn(cfg.H, cfg.C, cfg.d, generator=g, device=self.device)
        self.concepts = concepts / concepts.norm(dim=-1, keepdim=True) * (cfg.d ** 0.5)
        self._gen = g

    def hyperplanes(self) -> torch.Tensor:
        return draw_cross_hyperplanes(self.cfg.nbits, self.cfg.d, self.cfg.seed)

    def prompt(self):
        cfg, g = self.cfg, self._gen
        idx = torch.arange(cfg.L, device=self.device) % cfg.C
        K = self.concepts[:, idx, :] + cfg.sigma * torch.randn(cfg.H, cfg.L, cfg.d, generator=g, device=self.device)
        V = torch.randn(cfg.L, cfg.H, cfg.d, generator=g, device=self.device)
        return K.transpose(0, 1).contiguous().to(torch.bfloat16), V.to(torch.bfloat16)

    def self_qkv(self, call: int):
        """Self-attention projections Q, K, V [F*P, H, d] of the block of call `call`:
        N(0, 1) draws rounded to bf16 (the buckets come from the cross-attention queries)."""
        cfg = self.cfg
        g = torch.Generator(device=self.device).manual_seed((cfg.seed * 7_000_003 + call * 104_729 + 11) % (2 ** 62))
        return tuple(torch.randn(cfg.T, cfg.H, cfg.d, generator=g, device=self.device).to(torch.bfloat16)
                     for _ in range(3))

    def queries(self, call: int) -> torch.Tensor:
        cfg = self.cfg
        g = torch.Generator(device=self.device).manual_seed((cfg.seed * 1_000_003 + call * 7919 + 3) % (2 ** 62))
        frames = []
        for _ in range(cfg.F):
            shown = torch.randperm(cfg.C, generator=g, device=self.device)[: cfg.A]
            pick = shown[torch.randint(0, cfg.A, (cfg.P,), generator=g, device=self.device)]
            q = self.concepts[:, pick, :]                          # [H, P, d]
            q = q + cfg.sigma * torch.randn(cfg.H, cfg.P, cfg.d, generator=g, device=self.device)
            frames.append(q.transpose(0, 1))
        return torch.cat(frames, dim=0).contiguous().to(torch.bfloat16)
