"""Synthetic workload table for the Prism block-sparse video self-attention path.

Each entry fixes the latent grid, the attention shape, the storage dtype, the
selection parameters (Top-k, Top-p) and the recipe of the seeded input
generator (``inputs.py``).  The grids are the latent shapes the Prism pages
quote for 720p / 1080p / 2K clips ("Prism: Dynamic Sparse Attention for Native
2K Joint Video-Audio Generation Model Training", Problem & motivation: a 2K clip
gives hundreds of thousands to over a million tokens; FAQ 1: a 10 s 2K clip has
more than 870k video tokens).  No dataset is used; every tensor is synthetic.

This module holds no arithmetic of the method.
"""
from __future__ import annotations

from dataclasses import dataclass, field, asdict


@dataclass(frozen=True)
class PrismConfig:
    name: str
    T: int
    H: int
    W: int
    heads: int
    head_dim: int
    dtype: str              # "f32" or "bf16": storage dtype of Q, K, V, dO, h_hat
    top_k: int
    top_p: float
    gen: str                # "aniso" (per-zone 1-D smoothing) or "fgbg" (foreground/background)
    alpha: float            # weight of the smooth component added to Q, K (and V for "aniso")
    n_blobs: tuple          # (min, max) number of sound-source blobs in h_hat
    seed: int
    audio_dim: int = 64
    aniso_sigma: float = 3.0
    fg_frac: float = 0.2
    bg_sigma: float = 4.0
    blob_sigma: float = 3.0
    blob_amp: float = 3.0
    hhat_noise_std: float = 0.1

    @property
    def n_tokens(self) -> int:
        return self.T * self.H * self.W

    @property
    def n_zones(self) -> int:
        return self.n_tokens // 512

    def to_dict(self) -> dict:
        return asdict(self)


_BASE_SEED = 20261004

CONFIGS = {
    # 8x16x16 grid, 2048 tokens, 4 zones; small enough for the fp64 oracle in full.
    "tiny": PrismConfig("tiny", 8, 16, 16, heads=2, head_dim=64, dtype="f32",
                        top_k=4, top_p=0.9, gen="aniso", alpha=1.5, n_blobs=(1, 1),
                        seed=_BASE_SEED + 0),
    "720p": PrismConfig("720p", 16, 48, 80, heads=24, head_dim=128, dtype="bf16",
                        top_k=8, top_p=0.9, gen="aniso", alpha=1.5, n_blobs=(1, 3),
                        seed=_BASE_SEED + 100),
    "1080p": PrismConfig("1080p", 24, 72, 120, heads=24, head_dim=128, dtype="bf16",
                         top_k=8, top_p=0.9, gen="aniso", alpha=1.5, n_blobs=(3, 3),
                         seed=_BASE_SEED + 200),
    # headline: 32x72x128 grid, 294,912 tokens, 576 zones
    "2k": PrismConfig("2k", 32, 72, 128, heads=24, head_dim=128, dtype="bf16",
                      top_k=8, top_p=0.9, gen="fgbg", alpha=1.5, n_blobs=(4, 4),
                      seed=_BASE_SEED + 300),
    # 112x72x128 grid, 1,032,192 tokens: nearly isotropic Q/K, Top-p expands widely
    "long": PrismConfig("long", 112, 72, 128, heads=24, head_dim=128, dtype="bf16",
                        top_k=8, top_p=0.95, gen="fgbg", alpha=0.3, n_blobs=(6, 6),
                        seed=_BASE_SEED + 400),
}


def get_config(name: str, **overrides) -> PrismConfig:
    """Return a config by name, optionally with fields replaced (e.g. a smaller grid)."""
    cfg = CONFIGS[name]
    if overrides:
        d = cfg.to_dict()
        d.update(overrides)
        d["n_blobs"] = tuple(d["n_blobs"])
        cfg = PrismConfig(**d)
    for ax in (cfg.T, cfg.H, cfg.W):
        if ax <= 0 or ax % 8:
            raise ValueError(f"grid axes must be positive multiples of 8, got {cfg.T}x{cfg.H}x{cfg.W}")
    return cfg
