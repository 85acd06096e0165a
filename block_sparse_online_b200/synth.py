"""Seeded synthetic spatio-temporal Q/K/V for the Sol-Attn forward operator.

This module only makes inputs. It holds none of the operator's arithmetic
(no pooling, proxy, threshold or attention), so both the CUDA path and the
fp64 oracle can consume exactly the same bf16 bits.

The pages evaluate on DiT video/image models (Wan2.1, HunyuanVideo, Bernini,
Ideogram 4) whose weights and benchmark prompts are not available here. The
generator stands in for their self-attention inputs: tokens are the cells of a
(t, y, x) patch grid flattened t-major, and Q and K share a smooth positional
projection so that attention is local in space and time, which is the property
the method exploits (Sol-Attn, ai-feeds summary, "局限" (limitations): the
method relies on locality in the attention maps of video diffusion models).

Recipe (per batch element b and head h, all draws from
``numpy.random.Generator(PCG64(SeedSequence([seed, b, h])))``):

* phi(t, y, x): 96 features = for each axis a in (t, y, x) with length L_a and
  16 frequencies w_f = pi * L_a ** (-f / 15) (f = 0..15; pi * 2 ** -f for a
  length-1 axis), the values sin(w_f * coord) and cos(w_f * coord).
* W ~ N(0, 1/96) of shape [96, d], shared by Q and K; Wv ~ N(0, 1/96).
* Q = c * phi W + 0.5 * N(0, 1), K = c * phi W + 0.5 * N(0, 1) (independent
  noise), V = N(0, 1) + phi Wv.
* c >= 0 is found by bisection so that the standard deviation of the logits
  q.k / sqrt(d) over 4096 seeded random token pairs equals the head's target
  alpha (the noise alone gives about 0.25; smaller targets clamp c = 0).
* The float32 result is rounded once to bf16 (round to nearest even).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

INF = float("inf")


@dataclass(frozen=True)
class Config:
    name: str
    B: int
    H: int
    d: int
    grid: tuple  # (T, Y, X)
    Bq: int
    Bk: int
    taus: tuple
    seed: int
    modes: tuple = ("dense", "keep_drop", "keep_correct")
    alpha: float = 3.0
    alpha_range: tuple | None = None     # per-head alpha ~ U[lo, hi]
    uniform_heads_frac: float = 0.0      # fraction of heads given alpha_uniform
    alpha_uniform: float = 0.3
    note: str = field(default="", compare=False)

    @property
    def N(self) -> int:
        T, Y, X = self.grid
        return T * Y * X

    @property
    def nQB(self) -> int:
        return -(-self.N // self.Bq)

    @property
    def nKB(self) -> int:
        return -(-self.N // self.Bk)

    def dense_flops(self) -> float:
        """4 B H N^2 d: the two matmuls of dense attention, 2 flops per MAC."""
        return 4.0 * self.B * self.H * self.N * self.N * self.d

    def shape(self):
        return (self.B, self.H, self.N, self.d)


CONFIGS = {
    "tiny": Config("tiny", B=1, H=2, d=64, grid=(4, 16, 16), Bq=64, Bk=64,
                   taus=(2.0, 4.0, INF), seed=1000,
                   note="B=1 H=2 d=64 N=1024 (4x16x16), blocks 64x64"),
    "image": Config("image", B=8, H=16, d=128, grid=(1, 64, 64), Bq=64, Bk=64,
                    taus=(2.0, 4.0, 6.0, INF), seed=1001,
                    note="image-DiT shaped: B=8 H=16 d=128 N=4096 (1x64x64), blocks 64x64"),
    "video480": Config("video480", B=1, H=12, d=128, grid=(21, 30, 52), Bq=128, Bk=128,
                       taus=(2.0, 3.0, 4.0, 6.0, INF), seed=1002,
                       note="480p video shaped: B=1 H=12 d=128 N=32760 (21x30x52), blocks 128x128, tail 120"),
    "video720": Config("video720", B=1, H=24, d=128, grid=(21, 45, 80), Bq=128, Bk=128,
                       taus=(3.0, 4.0, 6.0), seed=1003, alpha_range=(1.5, 4.0),
                       note="720p video shaped: B=1 H=24 d=128 N=75600 (21x45x80), blocks 128x128, tail 80"),
    "long": Config("long", B=1, H=24, d=128, grid=(33, 45, 80), Bq=128, Bk=128,
                   taus=(3.0, 4.0, 6.0, INF), seed=1004, uniform_heads_frac=0.05,
                   note="long video: B=1 H=24 d=128 N=118800 (33x45x80), blocks 128x128, tail 16"),
}

N_FREQ = 16
N_FEAT = 6 * N_FREQ  # sin and cos for 16 frequencies on 3 axes
CALIB_PAIRS = 4096


def token_coords(grid):
    """(t, y, x) integer coordinates of the tokens, flattened t-major: n = (t*Y + y)*X + x."""
    T, Y, X = grid
    n = np.arange(T * Y * X, dtype=np.int64)
    return n // (Y * X), (n // X) % Y, n % X


def features(grid) -> np.ndarray:
    """phi: [N, 96] float64 sin/cos positional features of the grid."""
    cols = []
    f = np.arange(N_FREQ, dtype=np.float64)
    for coord, L in zip(token_coords(grid), grid):
        if L > 1:
            omega = math.pi * np.power(float(L), -f / (N_FREQ - 1))
        else:
            omega = math.pi * np.power(2.0, -f)
        ang = coord.astype(np.float64)[:, None] * omega[None, :]
        cols.append(np.sin(ang))
        cols.append(np.cos(ang))
    return np.concatenate(cols, axis=1)


def head_alphas(cfg: Config) -> np.ndarray:
    """Target logit std per (b, h): [B, H] float64."""
    alphas = np.full((cfg.B, cfg.H), cfg.alpha, dtype=np.float64)
    if cfg.alpha_range is not None:
        rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([cfg.seed, 10_000])))
        lo, hi = cfg.alpha_range
        alphas = rng.uniform(lo, hi, size=(cfg.B, cfg.H))
    if cfg.uniform_heads_frac > 0:
        rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([cfg.seed, 20_000])))
        n_uni = max(1, int(round(cfg.uniform_heads_frac * cfg.H)))
        for b in range(cfg.B):
            heads = rng.choice(cfg.H, size=n_uni, replace=False)
            alphas[b, heads] = cfg.alpha_uniform
    return alphas


def _calibrate(base, nq, nk, a_idx, b_idx, d, alpha):
    """Bisection for c >= 0 with std(q.k/sqrt(d)) over the sampled pairs == alpha."""
    ba, bb = base[a_idx], base[b_idx]
    na, nb = 0.5 * nq[a_idx].astype(np.float64), 0.5 * nk[b_idx].astype(np.float64)
    inv = 1.0 / math.sqrt(d)

    def std(c):
        return float(np.std(np.einsum("pd,pd->p", c * ba + na, c * bb + nb) * inv))

    if std(0.0) >= alpha:
        return 0.0
    hi = 1.0
    while std(hi) < alpha:
        hi *= 2.0
        if hi > 1e6:
            break
    lo = 0.0
    for _ in range(60):
        mid = 0.5 * (lo + hi)
        if std(mid) < alpha:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def make_head(cfg: Config, b: int, h: int, phi: np.ndarray, alpha: float):
    """One (b, h) slice: (q, k, v) float32 [N, d] before bf16 rounding."""
    N, d = cfg.N, cfg.d
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([cfg.seed, b, h])))
    W = rng.standard_normal((N_FEAT, d)) / math.sqrt(N_FEAT)
    Wv = rng.standard_normal((N_FEAT, d)) / math.sqrt(N_FEAT)
    nq = rng.standard_normal((N, d), dtype=np.float32)
    nk = rng.standard_normal((N, d), dtype=np.float32)
    nv = rng.standard_normal((N, d), dtype=np.float32)
    a_idx = rng.integers(0, N, size=CALIB_PAIRS)
    b_idx = rng.integers(0, N, size=CALIB_PAIRS)
    base = phi @ W  # [N, d] float64
    c = _calibrate(base, nq, nk, a_idx, b_idx, d, alpha)
    q = (c * base + 0.5 * nq).astype(np.float32)
    k = (c * base + 0.5 * nk).astype(np.float32)
    v = (nv + phi @ Wv).astype(np.float32)
    return q, k, v


def make_inputs(cfg: Config | str, device="cpu"):
    """(q, k, v) bf16 tensors [B, H, N, d] on ``device`` for a named config."""
    if isinstance(cfg, str):
        cfg = CONFIGS[cfg]
    phi = features(cfg.grid)
    alphas = head_alphas(cfg)
    shape = cfg.shape()
    q = torch.empty(shape, dtype=torch.bfloat16)
    k = torch.empty(shape, dtype=torch.bfloat16)
    v = torch.empty(shape, dtype=torch.bfloat16)
    for b in range(cfg.B):
        for h in range(cfg.H):
            qh, kh, vh = make_head(cfg, b, h, phi, float(alphas[b, h]))
            q[b, h] = torch.from_numpy(qh).to(torch.bfloat16)
            k[b, h] = torch.from_numpy(kh).to(torch.bfloat16)
            v[b, h] = torch.from_numpy(vh).to(torch.bfloat16)
    if device != "cpu":
        q, k, v = q.to(device), k.to(device), v.to(device)
    return q, k, v


def make_random(B, H, N, d, seed=0, scale=1.0, device="cpu"):
    """Plain N(0, scale^2) bf16 Q/K and N(0,1) V, for edge-case shapes."""
    g = torch.Generator().manual_seed(seed)
    q = (torch.randn((B, H, N, d), generator=g) * scale).to(torch.bfloat16)
    k = (torch.randn((B, H, N, d), generator=g) * scale).to(torch.bfloat16)
    v = torch.randn((B, H, N, d), generator=g).to(torch.bfloat16)
    if device != "cpu":
        q, k, v = q.to(device), k.to(device), v.to(device)
    return q, k, v


def small_config(name="small", N=1000, d=64, H=2, B=1, Bq=64, Bk=64, grid=None, seed=7, alpha=3.0):
    """An ad-hoc small config on a grid with the same generator (for parity tests)."""
    if grid is None:
        grid = (1, 1, N)
    return Config(name, B=B, H=H, d=d, grid=grid, Bq=Bq, Bk=Bk, taus=(2.0, 4.0, INF),
                  seed=seed, alpha=alpha)
