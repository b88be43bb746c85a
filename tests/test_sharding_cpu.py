"""The head-sharded zone indicator's exchange on CPU: two gloo ranks, each
holding half the heads, form their per-zone partial sums over their own
channels (from the oracle, standing in for prism_zone_partials, which needs a
GPU) and add them with the product's reduce_zone_partials; the result must be
the full-channel statistics of the oracle on every rank."""
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as orc
from dynamic_block_sparse_macro_b200.sharding import head_slice, reduce_zone_partials

T, H, W, HEADS, DH, DA = 8, 16, 16, 6, 4, 8


def _inputs():
    rng = np.random.default_rng(31)
    V = rng.normal(size=(T * H * W, HEADS, DH))
    V += np.linspace(0, 3, T)[:, None, None, None].repeat(H * W, 1).reshape(-1, 1, 1) * rng.normal(size=(HEADS, DH))
    hh = rng.normal(size=(T * H * W, DA)) * 0.1
    return V, hh


def _partials(V, hh):
    """[2, Z, 4]: un-normalised video sums over V's channels, and the audio statistics."""
    D = V.shape[1] * V.shape[2]
    ind = orc.zone_indicator(V, hh, T, H, W)
    video = np.concatenate([8.0 * D * ind["sigma2_v"], 512.0 * D * ind["rho_raw"][:, None]], axis=1)
    audio = np.concatenate([ind["A"][:, None], ind["sigma2_a"]], axis=1)
    return np.stack([video, audio])


def _rank(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        V, hh = _inputs()
        sl = head_slice(HEADS, rank, world)
        p = torch.from_numpy(_partials(V[:, sl, :], hh).copy())
        Z = p.shape[1]
        reduce_zone_partials(p, Z)
        out[rank] = p.numpy()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_two_ranks_recover_the_full_channel_statistics(world):
    port = 29611 + world
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank, args=(world, port, out), nprocs=world, join=True)
        got = [out[r] for r in range(world)]
    V, hh = _inputs()
    full = _partials(V, hh)
    for r in range(world):
        np.testing.assert_allclose(got[r], full, rtol=1e-12, atol=1e-12)


def test_head_slices_cover_every_head_once():
    for heads in (1, 2, 5, 24):
        for world in range(1, heads + 1):
            sl = [head_slice(heads, r, world) for r in range(world)]
            assert [h for s in sl for h in range(s.start, s.stop)] == list(range(heads))
            sizes = [s.stop - s.start for s in sl]
            assert max(sizes) - min(sizes) <= 1
