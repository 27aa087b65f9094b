"""Seeded synthetic workloads shaped like autoregressive video-diffusion attention layers.

FAST-AR's TempCache is measured on video models and benchmark suites that are not
available here (FAST-AR summary, "Resultados Principais"), so every input is drawn
from a seeded generator that imitates the structure the method exploits: keys that
change slowly from frame to frame (FAST-AR summary, section 1, "temporal key
redundancy").

Recipe, per head:
  * S prototypes drawn from N(0, I_d) and rescaled to norm sqrt(d);
  * frame 0: every one of the P token positions draws a prototype uniformly;
  * each later frame: a position keeps its previous prototype with probability
    p_stay, else it draws a new one uniformly;
  * key = prototype + N(0, sigma^2 I_d); values ~ N(0, 1); queries ~ N(0, 1),
    drawn afresh for every attention call;
  * bf16 workloads round every draw to bf16 (round to nearest even) before
    either implementation sees it; the f32 workload keeps fp32.
Hyperplanes for the sign-of-random-projection hash are N(0, 1) draws rounded to
bf16 values, one set shared by all heads.

A chunk holds F consecutive frames, T = P*F tokens, token t = f*P + p. Tensors are
token-major: K, V, Q are [T, H, d].

Nothing here implements the method: it only draws numbers.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class WorkloadConfig:
    name: str
    H: int          # heads
    d: int          # head dimension
    P: int          # tokens per frame
    F: int          # frames per chunk
    chunks: int     # chunks in the rollout
    attends: int    # attention calls per chunk
    S: int          # prototypes per head
    p_stay: float   # probability that a position keeps its prototype
    sigma: float    # key noise standard deviation
    nbits: int      # hash bits
    tau: float      # cosine merge threshold
    dtype: str      # "bf16" or "f32" storage
    capacity: int   # cache entries per head
    seed: int

    @property
    def T(self) -> int:
        return self.P * self.F

    def replace(self, **kw) -> "WorkloadConfig":
        return dataclasses.replace(self, **kw)


# The five workloads: tiny fp32; Wan-2.1-1.3B-shaped layer; long rollout (and its
# exact-duplicate variant); Wan-14B 720p-shaped layer; low-redundancy stress.
# Capacities not fixed by the workload description are the total number of
# tokens appended, so that no commit can overflow.
CONFIGS = {
    "tiny-f32": WorkloadConfig("tiny-f32", 1, 64, 64, 1, 16, 4, 128, 0.8, 0.05, 8, 0.95, "f32", 1024, 1000),
    "wan1.3b": WorkloadConfig("wan1.3b", 12, 128, 1560, 3, 40, 4, 4096, 0.8, 0.05, 16, 0.95, "bf16", 187200, 1001),
    "long-rollout": WorkloadConfig("long-rollout", 12, 128, 1560, 3, 160, 4, 4096, 0.9, 0.05, 16, 0.95, "bf16", 748800, 1002),
    "long-rollout-dup": WorkloadConfig("long-rollout-dup", 12, 128, 1560, 3, 160, 4, 4096, 0.9, 0.0, 16, 1.0 - 1e-6, "bf16", 748800, 1012),
    "wan14b-720p": WorkloadConfig("wan14b-720p", 40, 128, 3600, 3, 80, 4, 16384, 0.8, 0.05, 16, 0.95, "bf16", 864000, 1003),
    "low-redundancy": WorkloadConfig("low-redundancy", 12, 128, 1560, 3, 100, 4, 65536, 0.3, 0.08, 18, 0.95, "bf16", 262144, 1004),
}


def round_to_bf16(x: torch.Tensor) -> torch.Tensor:
    """Round fp32 draws to the nearest bf16 value (ties to even); returns fp32."""
    return x.to(torch.float32).to(torch.bfloat16).to(torch.float32)


def draw_hyperplanes(nbits: int, d: int, seed: int) -> torch.Tensor:
    """N(0,1) hyperplane normals rounded to bf16 values, [nbits, d] fp32 on the CPU."""
    g = torch.Generator(device="cpu").manual_seed(int(seed) * 7919 + 17)
    return round_to_bf16(torch.randn(nbits, d, generator=g, dtype=torch.float32))


class Workload:
    """Iterates the chunks of one synthetic rollout.

    `next_chunk()` returns (K, V) as [T, H, d] tensors in the storage dtype
    (torch.bfloat16 or torch.float32) on `device`; `queries(c, a)` returns the
    queries of attention call `a` of chunk `c`. The generator is deterministic
    for a given (config, device).
    """

    def __init__(self, cfg: WorkloadConfig, device="cpu"):
        self.cfg = cfg
        self.device = torch.device(device)
        self.storage = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
        self._gen = torch.Generator(device=self.device).manual_seed(cfg.seed)
        H, S, d = cfg.H, cfg.S, cfg.d
        protos = torch.randn(H, S, d, generator=self._gen, device=self.device)
        protos = protos / protos.norm(dim=-1, keepdim=True) * (d ** 0.5)
        self.protos = protos
        self._idx = None          # [H, P] current prototype of each position
        self.chunk_index = 0

    @property
    def T(self) -> int:
        return self.cfg.T

    def hyperplanes(self) -> torch.Tensor:
        return draw_hyperplanes(self.cfg.nbits, self.cfg.d, self.cfg.seed)

    def _store(self, x: torch.Tensor) -> torch.Tensor:
        return x.to(self.storage).contiguous()

    def _next_frame_keys(self) -> torch.Tensor:
        cfg, g, dev = self.cfg, self._gen, self.device
        H, P, S = cfg.H, cfg.P, cfg.S
        fresh = torch.randint(0, S, (H, P), generator=g, device=dev)
        if self._idx is None:
            self._idx = fresh
        else:
            stay = torch.rand(H, P, generator=g, device=dev) < cfg.p_stay
            self._idx = torch.where(stay, self._idx, fresh)
        base = torch.gather(self.protos, 1, self._idx[:, :, None].expand(H, P, cfg.d))  # [H,P,d]
        if cfg.sigma > 0:
            base = base + cfg.sigma * torch.randn(H, P, cfg.d, generator=g, device=dev)
        return base.transpose(0, 1)  # [P, H, d]

    def next_chunk(self):
        cfg = self.cfg
        frames = [self._next_frame_keys() for _ in range(cfg.F)]
        K = torch.cat(frames, dim=0)  # [T, H, d], frame-major
        V = torch.randn(cfg.T, cfg.H, cfg.d, generator=self._gen, device=self.device)
        self.chunk_index += 1
        return self._store(K), self._store(V)

    def queries(self, chunk: int, call: int, rows: int | None = None) -> torch.Tensor:
        cfg = self.cfg
        g = torch.Generator(device=self.device).manual_seed(
            (cfg.seed * 1_000_003 + chunk * 1009 + call * 17 + 5) % (2 ** 62))
        n = cfg.T if rows is None else rows
        Q = torch.randn(n, cfg.H, cfg.d, generator=g, device=self.device)
        return self._store(Q)
