"""Seeded synthetic inputs for head-wise dynamic sparse global attention.

This module only draws inputs: token layouts, the five named workloads, and the
Q/K/V/DINO tensors built from a latent scene.  It contains none of the
attention method's arithmetic (no selection, no softmax, no scoring), so both
the CPU oracle and the CUDA path can consume its output without sharing code.

Workloads (shapes follow the SAF3R paper's dense long-sequence setting, section
5.1 "Evaluation benchmarks": 300-700 frames of 37x37 patches plus camera and
register tokens; the paper's datasets are not used, synthetic tokens stand in):

  tiny   S=4   views, 16x16 patches, H=4  (one head of each kind)
  s32    S=32  views, 37x37 patches, H=16
  s100   S=100 views, 37x37 patches, H=16, 4 layer calls reuse one index cache
  s200   S=200 views, 37x37 patches, H=16
  stack  S=64  views, 37x37 patches, H=16, 24 layers, per-head profiling

Token recipe (per view s, patch p):  x = A z[(p + delta*s) mod M] + 0.3 eps,
special tokens ~ N(0, I_D);  Q/K/V = x W (W ~ N(0, 1/D)), rounded to bf16;
DINO feature = normalize(B z[...] + 0.2 eps'), fp32.  Every random stream is a
PCG64 generator keyed by (seed, component, index), so any view or layer can be
regenerated alone and the draw order never depends on chunking.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np

# head kinds (paper section 3, Observation #2; kernels of section 4.1)
POSITION, PROBE, CORR, SCAN, DENSE, HYBRID, TOKEN = 0, 1, 2, 3, 4, 5, 6
KIND_NAMES = {POSITION: "position", PROBE: "probe", CORR: "corr", SCAN: "scan", DENSE: "dense", HYBRID: "hybrid",
              TOKEN: "token"}

N_SPECIAL = 5      # 1 camera + 4 register tokens per view
HEAD_DIM = 64
DINO_DIM = 384
TILE = 64


@dataclass(frozen=True)
class Layout:
    """Token layout of one global-attention layer.

    Per view: the 5 special tokens first (camera, then 4 registers), then the
    g*g patch tokens in raster order.  Token t = s*V + i.
    """
    S: int
    g: int
    H: int
    d: int = HEAD_DIM
    n_special: int = N_SPECIAL
    dino_dim: int = DINO_DIM
    tile: int = TILE

    @property
    def P(self) -> int:
        return self.g * self.g

    @property
    def V(self) -> int:
        return self.P + self.n_special

    @property
    def N(self) -> int:
        return self.S * self.V

    @property
    def T(self) -> int:
        return (self.N + self.tile - 1) // self.tile


@dataclass(frozen=True)
class HeadCfg:
    kind: int
    k: int = 0          # probe: number of patch keys; corr: number of key tiles
    stride: int = 0     # scan
    phase: int = 0      # scan
    radius: int = 1     # position


@dataclass
class Workload:
    name: str
    layout: Layout
    M: int              # latent scene points
    delta: int          # per-view shift of the latent index
    D: int              # token width
    heads: List[HeadCfg]
    calls: int = 1      # layer calls that share one index cache
    sample_rows: int = 0  # query rows per head the oracle checks (0 = all)
    seed: int = 0
    layers: int = 1
    candidates: List[HeadCfg] = field(default_factory=list)


def _split16(probe_k: int, corr_k: int, stride: int) -> List[HeadCfg]:
    heads = [HeadCfg(POSITION) for _ in range(4)]
    heads += [HeadCfg(PROBE, k=probe_k) for _ in range(4)]
    heads += [HeadCfg(CORR, k=corr_k) for _ in range(4)]
    heads += [HeadCfg(SCAN, stride=stride, phase=h % stride) for h in range(12, 16)]
    return heads


def _profile_candidates() -> List[HeadCfg]:
    """The ten per-head candidates of the profiled stack (a scan candidate's
    phase is replaced by head index mod stride when it is applied to a head)."""
    c = [HeadCfg(POSITION)]
    c += [HeadCfg(PROBE, k=k) for k in (2048, 4096, 8192)]
    c += [HeadCfg(CORR, k=k) for k in (16, 32, 64)]
    c += [HeadCfg(SCAN, stride=s, phase=0) for s in (8, 16, 32)]
    return c


SEED_BASE = 20260703

WORKLOADS = {
    "tiny": Workload("tiny", Layout(S=4, g=16, H=4), M=512, delta=37, D=256,
                     heads=[HeadCfg(POSITION), HeadCfg(PROBE, k=128), HeadCfg(CORR, k=4),
                            HeadCfg(SCAN, stride=8, phase=3)],
                     seed=SEED_BASE + 0),
    "s32": Workload("s32", Layout(S=32, g=37, H=16), M=4096, delta=97, D=1024,
                    heads=_split16(4096, 32, 10), seed=SEED_BASE + 1000, sample_rows=2048),
    "s100": Workload("s100", Layout(S=100, g=37, H=16), M=4096, delta=97, D=1024,
                     heads=_split16(8192, 64, 16), calls=4, sample_rows=2048,
                     seed=SEED_BASE + 2000),
    "s200": Workload("s200", Layout(S=200, g=37, H=16), M=4096, delta=97, D=1024,
                     heads=_split16(13740, 215, 20), sample_rows=1024, seed=SEED_BASE + 3000),
    # the S=32 layer with its position heads replaced by token-wise per-frame DINO Top-16 heads
    "s32_token": Workload("s32_token", Layout(S=32, g=37, H=16), M=4096, delta=97, D=1024,
                          heads=[HeadCfg(TOKEN, k=16)] * 4 + _split16(4096, 32, 10)[4:],
                          sample_rows=256, seed=SEED_BASE + 1000),
    # the S=100 layer with its position heads replaced by token-wise per-frame DINO Top-16 heads
    "s100_token": Workload("s100_token", Layout(S=100, g=37, H=16), M=4096, delta=97, D=1024,
                           heads=[HeadCfg(TOKEN, k=16)] * 4 + _split16(8192, 64, 16)[4:],
                           calls=4, sample_rows=128, seed=SEED_BASE + 2000),
    # the S=100 layer with its correspondence heads as tile Top-64 united with a stride-32 lattice
    "s100_hybrid": Workload("s100_hybrid", Layout(S=100, g=37, H=16), M=4096, delta=97, D=1024,
                            heads=_split16(8192, 64, 16)[:8] +
                            [HeadCfg(HYBRID, k=64, stride=32, phase=h % 32) for h in range(8, 12)] +
                            _split16(8192, 64, 16)[12:],
                            calls=4, sample_rows=2048, seed=SEED_BASE + 2000),
    "stack": Workload("stack", Layout(S=64, g=37, H=16), M=4096, delta=97, D=1024,
                      heads=_split16(4096, 32, 10), layers=24, sample_rows=256,
                      seed=SEED_BASE + 4000, candidates=_profile_candidates()),
}


def _rng(seed: int, *key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, *key])))


# component ids of the random streams
_Z, _A, _SPEC, _EPS, _B, _EPSD, _W = 1, 2, 3, 4, 5, 6, 7


class Scene:
    """The per-input part of a workload: latent points, token matrix, DINO features."""

    def __init__(self, wl: Workload, seed: Optional[int] = None):
        self.wl = wl
        self.seed = wl.seed if seed is None else seed
        L = wl.layout
        self.z = _rng(self.seed, _Z).standard_normal((wl.M, 64), dtype=np.float32)
        self.A = (_rng(self.seed, _A).standard_normal((wl.D, 64), dtype=np.float32)
                  * np.float32(1.0 / 8.0))
        self.B = (_rng(self.seed, _B).standard_normal((L.dino_dim, 64), dtype=np.float32)
                  * np.float32(1.0 / 8.0))
        self._x = None
        self._dino = None

    def latent_index(self, s: int) -> np.ndarray:
        L = self.wl.layout
        return (np.arange(L.P) + self.wl.delta * s) % self.wl.M

    def tokens(self) -> np.ndarray:
        """fp32 [N][D] token matrix (built once)."""
        if self._x is None:
            wl, L = self.wl, self.wl.layout
            x = np.empty((L.N, wl.D), dtype=np.float32)
            za = self.z @ self.A.T                      # [M][D]
            for s in range(L.S):
                base = s * L.V
                x[base:base + L.n_special] = _rng(self.seed, _SPEC, s).standard_normal(
                    (L.n_special, wl.D), dtype=np.float32)
                eps = _rng(self.seed, _EPS, s).standard_normal((L.P, wl.D), dtype=np.float32)
                x[base + L.n_special:base + L.V] = za[self.latent_index(s)] + np.float32(0.3) * eps
            self._x = x
        return self._x

    def dino(self) -> np.ndarray:
        """fp32 [S*P][dino_dim] L2-normalised DINO-like patch features."""
        if self._dino is None:
            L = self.wl.layout
            f = np.empty((L.S * L.P, L.dino_dim), dtype=np.float32)
            zb = self.z @ self.B.T                      # [M][dino_dim]
            for s in range(L.S):
                eps = _rng(self.seed, _EPSD, s).standard_normal((L.P, L.dino_dim), dtype=np.float32)
                blk = zb[self.latent_index(s)] + np.float32(0.2) * eps
                blk /= np.linalg.norm(blk, axis=1, keepdims=True).astype(np.float32)
                f[s * L.P:(s + 1) * L.P] = blk
            self._dino = f
        return self._dino


def projections(wl: Workload, seed: int, layer: int):
    """W_q, W_k, W_v of one layer, each fp32 [D][H*64] ~ N(0, 1/D)."""
    L = wl.layout
    sc = np.float32(1.0 / math.sqrt(wl.D))
    return [_rng(seed, _W, layer, which).standard_normal((wl.D, L.H * L.d), dtype=np.float32) * sc
            for which in range(3)]


def qkv(scene: Scene, layer: int = 0, device: str = "cpu"):
    """Q, K, V of one layer as torch bf16 tensors [H][N][64] on `device`.

    The projection runs as an fp32 matmul (torch, on `device`) and is rounded
    to bf16 with round-to-nearest-even.  Consumers that compare against each
    other must use the same returned tensors.
    """
    import torch
    wl, L = scene.wl, scene.wl.layout
    x = torch.from_numpy(scene.tokens()).to(device)
    out = []
    for w in projections(wl, scene.seed, layer):
        y = x @ torch.from_numpy(w).to(device)                 # [N][H*64] fp32
        y = y.view(L.N, L.H, L.d).transpose(0, 1).contiguous()  # [H][N][64]
        out.append(y.to(torch.bfloat16))
        del y
    return out


def bf16_to_f32(t) -> np.ndarray:
    """Exact fp32 numpy copy of a torch bf16 tensor (any device)."""
    import torch
    return t.detach().to("cpu").to(torch.float32).numpy()


def sample_rows(wl: Workload, head: int, n: int, seed_extra: int = 0) -> np.ndarray:
    """Seeded, sorted, distinct query rows of one head that the oracle checks.

    The sample always contains the first and last token, a special token and the
    first patch token of the last view, so tails and view borders are covered.
    """
    L = wl.layout
    if n <= 0 or n >= L.N:
        return np.arange(L.N)
    rng = _rng(wl.seed, 99, head, seed_extra)
    fixed = np.array([0, 1, L.N - 1, (L.S - 1) * L.V, (L.S - 1) * L.V + L.n_special], dtype=np.int64)
    pick = rng.choice(L.N, size=n, replace=False)
    return np.unique(np.concatenate([fixed, pick]))
