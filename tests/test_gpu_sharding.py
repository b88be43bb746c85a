"""Head-sharded zone indicator on one GPU: ranks are emulated one after
another (each computes prism_zone_partials over its own heads; the sum of
their video partials stands in for the all-reduce), then prism_zone_finalize.
The result must match the unsharded indicator (up to the order of the fp32
sums) and the oracle on the full channel set."""
import numpy as np
import pytest
import torch

import oracle as orc
from dynamic_block_sparse_macro_b200 import _abi, inputs
from dynamic_block_sparse_macro_b200.configs import get_config
from dynamic_block_sparse_macro_b200.sharding import ShardedZoneIndicator, head_slice

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,kw,world", [("2k", dict(T=16, H=24, W=32, heads=6), 2),
                                           ("2k", dict(T=16, H=24, W=32, heads=6), 3),
                                           ("tiny", {}, 2)])
def test_emulated_ranks_match_the_whole_indicator(name, kw, world):
    cfg = get_config(name, **kw)
    x = inputs.make_inputs(cfg, "cuda", with_grad=False)
    prob = _abi.problem(cfg.T, cfg.H, cfg.W, cfg.heads, cfg.head_dim, cfg.audio_dim, cfg.dtype)
    sz = _abi.query_sizes(prob)
    Z = int(sz.n_zones)
    f32 = dict(dtype=torch.float32, device="cuda")
    ref = {k: torch.empty(s, **f32) for k, s in (("g", (Z, 3)), ("rho", (Z,)), ("abar", (Z,)), ("zs", (Z, 8)))}
    ws = torch.empty(sz.ws_indicator, dtype=torch.uint8, device="cuda")
    _abi.prism_zone_indicator(prob, x["V"], x["hhat"], 1e-6, ref["g"], ref["rho"], ref["abar"], ref["zs"], ws)

    total = None
    for r in range(world):
        sl = head_slice(cfg.heads, r, world)
        Vl = x["V"][:, sl, :].contiguous()
        pl = _abi.problem(cfg.T, cfg.H, cfg.W, sl.stop - sl.start, cfg.head_dim, cfg.audio_dim, cfg.dtype)
        wl = torch.empty(_abi.query_sizes(pl).ws_indicator, dtype=torch.uint8, device="cuda")
        part = torch.empty((2, Z, 4), **f32)
        _abi.prism_zone_partials(pl, Vl, x["hhat"], part, wl)
        if total is None:
            total = part.clone()
        else:
            torch.testing.assert_close(part[1], total[1], rtol=0, atol=0)   # audio: the same on every rank
            total[0] += part[0]
    out = {k: torch.empty_like(v) for k, v in ref.items()}
    fws = torch.empty(Z * 16, dtype=torch.uint8, device="cuda")
    _abi.prism_zone_finalize(prob, total, 1e-6, "joint", out["g"], out["rho"], out["abar"], out["zs"], fws)
    torch.cuda.synchronize()
    for k in ref:
        torch.testing.assert_close(out[k], ref[k], rtol=1e-5, atol=1e-6)
    ind = orc.zone_indicator(inputs.to_f64(x["V"]), inputs.to_f64(x["hhat"]), cfg.T, cfg.H, cfg.W)
    np.testing.assert_allclose(out["g"].cpu().double().numpy(), ind["g"], rtol=2e-5, atol=1e-6)
    np.testing.assert_allclose(out["rho"].cpu().double().numpy(), ind["rho"], rtol=2e-5, atol=1e-6)


def test_single_rank_module():
    # without a process group the module holds every head and needs no exchange
    cfg = get_config("tiny")
    x = inputs.make_inputs(cfg, "cuda", with_grad=False)
    mod = ShardedZoneIndicator(cfg.T, cfg.H, cfg.W, cfg.heads, cfg.head_dim, cfg.audio_dim, cfg.dtype)
    g, rho, abar, zs = mod(x["V"], x["hhat"])
    ind = orc.zone_indicator(inputs.to_f64(x["V"]), inputs.to_f64(x["hhat"]), cfg.T, cfg.H, cfg.W)
    np.testing.assert_allclose(g.cpu().double().numpy(), ind["g"], rtol=2e-5, atol=1e-6)
    np.testing.assert_allclose(abar.cpu().double().numpy(), ind["abar"], rtol=2e-5, atol=1e-6)
