"""Seeded synthetic inputs for the Prism block-sparse attention path.

The same bytes feed the CUDA path and the fp64 oracle: tensors are generated
once (on whatever device is given, with a seeded ``torch.Generator``), cast to
the storage dtype, and the oracle reads host copies of those stored values.

Tensors (batch 1):
  Q, K, V, dO : raster ``[N, heads, head_dim]`` (N = T*H*W, r = (t*H + h)*W + w)
  hhat        : raster ``[N, audio_dim]``, the cached audio-to-video
                cross-attention output of the previous layer (Prism, Method 1:
                the audio guidance is the L2 norm of this tensor per token).

Recipes (the smooth parts give the zone indicator and the block scores
something to find):
  "aniso": X = N(0,1) + alpha * F, F = N(0,1) smoothed by a 1-D Gaussian
           (sigma ``aniso_sigma``) along one seeded axis per 8x8x8 zone and
           renormalised to unit variance per channel.  Q and K of a head share F;
           V has its own F.
  "fgbg":  a seeded ``fg_frac`` of the zones is foreground (unfiltered N(0,1));
           the rest is background: N(0,1) smoothed by a unit-sum 3-D Gaussian
           (sigma ``bg_sigma``) and not renormalised, so its token variance is
           about 1/(2 sqrt(pi) sigma)^3.  Q and K add alpha * L, L a unit-variance
           3-D smoothed field shared by Q and K of a head (locality of the
           pooled block scores).
  hhat:    N(0, hhat_noise_std^2) per channel plus blobs
           blob_amp * exp(-|x - c|^2 / (2 blob_sigma^2)) * u, u a seeded
           unit-RMS vector, c uniform inside one seeded zone.
  dO:      N(0,1).

Smoothing truncates the Gaussian at 3 sigma and zero-pads the grid edges.
Sub-stream seeds: Q=1, K=2, V=3, hhat=4, dO=5, blobs=6, zone axes / fg mask=7,
shared smooth fields=8, added to the config seed.

This module holds no arithmetic of the method itself.
"""
from __future__ import annotations

import math

import torch

from .configs import PrismConfig

_SUB = {"Q": 1, "K": 2, "V": 3, "hhat": 4, "dO": 5, "blobs": 6, "zones": 7, "shared": 8}


def _gen(cfg: PrismConfig, stream: str, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(cfg.seed * 16 + _SUB[stream])
    return g


def _gauss_taps(sigma: float, device) -> torch.Tensor:
    r = int(math.ceil(3.0 * sigma))
    x = torch.arange(-r, r + 1, dtype=torch.float64)
    w = torch.exp(-0.5 * (x / sigma) ** 2)
    w = w / w.sum()
    return w.to(device=device, dtype=torch.float32)


def _smooth_axis(x: torch.Tensor, axis: int, taps: torch.Tensor) -> torch.Tensor:
    """Zero-padded 1-D convolution of a [T, H, W, C] field along one grid axis."""
    r = (taps.numel() - 1) // 2
    n = x.shape[axis]
    out = torch.zeros_like(x)
    for k in range(-r, r + 1):
        w = float(taps[k + r])
        lo_dst, hi_dst = max(0, -k), min(n, n - k)
        if hi_dst <= lo_dst:
            continue
        dst = out.narrow(axis, lo_dst, hi_dst - lo_dst)
        src = x.narrow(axis, lo_dst + k, hi_dst - lo_dst)
        dst.add_(src, alpha=w)
    return out


def _smooth3(x: torch.Tensor, sigma: float) -> torch.Tensor:
    taps = _gauss_taps(sigma, x.device)
    for ax in range(3):
        x = _smooth_axis(x, ax, taps)
    return x


def _unit_var(x: torch.Tensor) -> torch.Tensor:
    flat = x.reshape(-1, x.shape[-1])
    std = flat.std(dim=0).clamp_min(1e-12)
    return x / std


def _zone_axes(cfg: PrismConfig, device) -> torch.Tensor:
    g = _gen(cfg, "zones", device)
    zt, zh, zw = cfg.T // 8, cfg.H // 8, cfg.W // 8
    return torch.randint(0, 3, (zt, zh, zw), generator=g, device=device)


def _fg_mask(cfg: PrismConfig, device) -> torch.Tensor:
    g = _gen(cfg, "zones", device)
    zt, zh, zw = cfg.T // 8, cfg.H // 8, cfg.W // 8
    Z = zt * zh * zw
    n_fg = int(round(cfg.fg_frac * Z))
    order = torch.randperm(Z, generator=g, device=device)
    m = torch.zeros(Z, dtype=torch.bool, device=device)
    m[order[:n_fg]] = True
    return m.reshape(zt, zh, zw)


def _zone_expand(zmask: torch.Tensor) -> torch.Tensor:
    """[ZT, ZH, ZW] per-zone values -> [T, H, W, 1] per-token values."""
    z = zmask.repeat_interleave(8, 0).repeat_interleave(8, 1).repeat_interleave(8, 2)
    return z.unsqueeze(-1)


def _aniso_field(cfg: PrismConfig, g: torch.Generator, C: int, axes: torch.Tensor) -> torch.Tensor:
    dev = axes.device
    taps = _gauss_taps(cfg.aniso_sigma, dev)
    noise = torch.randn((cfg.T, cfg.H, cfg.W, C), generator=g, device=dev)
    out = torch.zeros_like(noise)
    ax_tok = _zone_expand(axes)
    for a in range(3):
        out = torch.where(ax_tok == a, _smooth_axis(noise, a, taps), out)
    return _unit_var(out)


def _fgbg_field(cfg: PrismConfig, g: torch.Generator, C: int, fg: torch.Tensor) -> torch.Tensor:
    dev = fg.device
    noise = torch.randn((cfg.T, cfg.H, cfg.W, C), generator=g, device=dev)
    smooth = _smooth3(noise, cfg.bg_sigma)
    return torch.where(_zone_expand(fg), noise, smooth)


def _storage_dtype(cfg: PrismConfig):
    return {"f32": torch.float32, "bf16": torch.bfloat16}[cfg.dtype]


def make_qkv(cfg: PrismConfig, device="cpu"):
    """Seeded Q, K, V as raster [N, heads, head_dim] tensors in the storage dtype."""
    dev = torch.device(device)
    dt = _storage_dtype(cfg)
    N, h, d = cfg.n_tokens, cfg.heads, cfg.head_dim
    gq, gk, gv, gs = (_gen(cfg, s, dev) for s in ("Q", "K", "V", "shared"))
    Q = torch.empty((N, h, d), dtype=dt, device=dev)
    K = torch.empty_like(Q)
    V = torch.empty_like(Q)
    if cfg.gen == "aniso":
        axes = _zone_axes(cfg, dev)
    else:
        fg = _fg_mask(cfg, dev)
    # one head at a time keeps the fp32 temporaries at N*d elements
    for hh in range(h):
        if cfg.gen == "aniso":
            Fqk = _aniso_field(cfg, gs, d, axes)
            Fv = _aniso_field(cfg, gv, d, axes)
            q = torch.randn((cfg.T, cfg.H, cfg.W, d), generator=gq, device=dev) + cfg.alpha * Fqk
            k = torch.randn((cfg.T, cfg.H, cfg.W, d), generator=gk, device=dev) + cfg.alpha * Fqk
            v = torch.randn((cfg.T, cfg.H, cfg.W, d), generator=gv, device=dev) + cfg.alpha * Fv
        elif cfg.gen == "fgbg":
            L = _unit_var(_smooth3(torch.randn((cfg.T, cfg.H, cfg.W, d), generator=gs, device=dev),
                                   cfg.bg_sigma))
            q = _fgbg_field(cfg, gq, d, fg) + cfg.alpha * L
            k = _fgbg_field(cfg, gk, d, fg) + cfg.alpha * L
            v = _fgbg_field(cfg, gv, d, fg)
        else:
            raise ValueError(cfg.gen)
        Q[:, hh, :] = q.reshape(N, d).to(dt)
        K[:, hh, :] = k.reshape(N, d).to(dt)
        V[:, hh, :] = v.reshape(N, d).to(dt)
    return Q, K, V


def make_hhat(cfg: PrismConfig, device="cpu") -> torch.Tensor:
    """Seeded cached A2V cross-attention output, raster [N, audio_dim]."""
    dev = torch.device(device)
    gn, gb = _gen(cfg, "hhat", dev), _gen(cfg, "blobs", dev)
    Da = cfg.audio_dim
    x = cfg.hhat_noise_std * torch.randn((cfg.T, cfg.H, cfg.W, Da), generator=gn, device=dev)
    lo, hi = cfg.n_blobs
    nb = int(torch.randint(lo, hi + 1, (1,), generator=gb, device=dev).item())
    zt, zh, zw = cfg.T // 8, cfg.H // 8, cfg.W // 8
    tt = torch.arange(cfg.T, device=dev, dtype=torch.float32).view(-1, 1, 1)
    hh = torch.arange(cfg.H, device=dev, dtype=torch.float32).view(1, -1, 1)
    ww = torch.arange(cfg.W, device=dev, dtype=torch.float32).view(1, 1, -1)
    for _ in range(nb):
        z = int(torch.randint(0, zt * zh * zw, (1,), generator=gb, device=dev).item())
        origin = torch.tensor([(z // (zh * zw)) * 8, ((z // zw) % zh) * 8, (z % zw) * 8],
                              dtype=torch.float32, device=dev)
        c = origin + 8.0 * torch.rand(3, generator=gb, device=dev)
        u = torch.randn(Da, generator=gb, device=dev)
        u = u / u.pow(2).mean().sqrt()
        r2 = (tt - c[0]) ** 2 + (hh - c[1]) ** 2 + (ww - c[2]) ** 2
        amp = cfg.blob_amp * torch.exp(-r2 / (2.0 * cfg.blob_sigma ** 2))
        x = x + amp.unsqueeze(-1) * u
    return x.reshape(cfg.n_tokens, Da).to(_storage_dtype(cfg))


def make_dout(cfg: PrismConfig, device="cpu") -> torch.Tensor:
    """Seeded upstream gradient dO, raster [N, heads, head_dim]."""
    dev = torch.device(device)
    g = _gen(cfg, "dO", dev)
    return torch.randn((cfg.n_tokens, cfg.heads, cfg.head_dim), generator=g,
                       device=dev).to(_storage_dtype(cfg))


def make_inputs(cfg: PrismConfig, device="cpu", with_grad=True) -> dict:
    Q, K, V = make_qkv(cfg, device)
    out = {"Q": Q, "K": K, "V": V, "hhat": make_hhat(cfg, device)}
    if with_grad:
        out["dO"] = make_dout(cfg, device)
    return out


def to_f64(x: torch.Tensor):
    """Host fp64 numpy copy of stored values (what the oracle reads)."""
    return x.detach().to("cpu").to(torch.float64).numpy()
