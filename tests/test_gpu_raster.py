"""Stages 4-6 straight from the raster layout (prism_block_pool_score_raster,
prism_sparse_attn_fwd_raster): the kernels apply the permutation inside their
loads and stores instead of copying Q, K, V into the blocked layout and O back.
The same rows meet the same arithmetic in the same order, so P, the selection
and O must equal, bit for bit, those of the blocked layer; that layer's O is
checked against the oracle by the parity tests, and here once more."""
import numpy as np
import pytest
import torch

import oracle as orc
from dynamic_block_sparse_macro_b200 import inputs
from dynamic_block_sparse_macro_b200.configs import get_config
from dynamic_block_sparse_macro_b200.layer import PrismSparseAttention

from gpu_parity import REL_L2, host, rel_l2, unpack_sel

pytestmark = pytest.mark.gpu


def _pair(cfg, top_k=None, top_p=None):
    kw = dict(with_backward=False)
    k = cfg.top_k if top_k is None else top_k
    p = cfg.top_p if top_p is None else top_p
    blocked = PrismSparseAttention(cfg.T, cfg.H, cfg.W, cfg.heads, cfg.head_dim, cfg.audio_dim, cfg.dtype, k, p, **kw)
    raster = PrismSparseAttention(cfg.T, cfg.H, cfg.W, cfg.heads, cfg.head_dim, cfg.audio_dim, cfg.dtype, k, p,
                                  raster=True, **kw)
    return blocked, raster


@pytest.mark.parametrize("name,kw,top_p", [
    ("720p", dict(T=8, H=16, W=16, heads=2), None),
    ("720p", dict(T=16, H=32, W=32, heads=3), None),
    ("720p", dict(T=16, H=32, W=32, heads=3, head_dim=64), None),
    ("2k", dict(T=16, H=24, W=32, heads=2), None),
    ("2k", dict(T=16, H=24, W=32, heads=2), 1.0),        # dense: long tiles split and combined
])
def test_raster_forward_matches_blocked_bits(name, kw, top_p):
    cfg = get_config(name, **kw)
    x = inputs.make_inputs(cfg, "cuda", with_grad=False)
    blocked, raster = _pair(cfg, top_p=top_p)
    Ob = blocked.forward(x["Q"], x["K"], x["V"], x["hhat"])
    Or = raster.forward(x["Q"], x["K"], x["V"], x["hhat"])
    torch.cuda.synchronize()
    assert raster.status() == 0
    assert torch.equal(raster.perm, blocked.perm)
    assert torch.equal(raster.P_view(), blocked.P_view())
    assert torch.equal(raster.gsel, blocked.gsel)
    assert torch.equal(Or, Ob)
    # and the oracle, under the layer's own selection
    nb = raster.num_blocks()
    bs = raster.blk_start[: nb + 1].cpu().numpy().astype(np.int64)
    perm = raster.perm.cpu().numpy().astype(np.int64)
    Qb, Kb, Vb = (orc.permute(host(x[k]), perm) for k in ("Q", "K", "V"))
    O_ref, _ = orc.sparse_attention_fwd(Qb, Kb, Vb, bs, unpack_sel(raster.sel, nb))
    assert rel_l2(host(Or), orc.unpermute(O_ref, perm)) <= REL_L2[cfg.dtype]


def test_raster_forward_full_2k_grid():
    cfg = get_config("2k")
    x = inputs.make_inputs(cfg, "cuda", with_grad=False)
    blocked, raster = _pair(cfg)
    Ob = blocked.forward(x["Q"], x["K"], x["V"], x["hhat"])
    del blocked
    Or = raster.forward(x["Q"], x["K"], x["V"], x["hhat"])
    torch.cuda.synchronize()
    assert raster.status() == 0
    assert torch.equal(Or, Ob)


@pytest.mark.parametrize("name,kw,top_p", [
    ("720p", dict(T=8, H=16, W=16, heads=2), None),
    ("720p", dict(T=16, H=32, W=32, heads=3), None),
    ("720p", dict(T=16, H=32, W=32, heads=3, head_dim=64), None),
    ("2k", dict(T=16, H=24, W=32, heads=2), None),
    ("2k", dict(T=16, H=24, W=32, heads=2), 1.0),        # dense: split tiles on both sides
])
def test_raster_training_matches_blocked_bits(name, kw, top_p):
    cfg = get_config(name, **kw)
    x = inputs.make_inputs(cfg, "cuda")
    p = cfg.top_p if top_p is None else top_p
    mk = lambda raster: PrismSparseAttention(cfg.T, cfg.H, cfg.W, cfg.heads, cfg.head_dim, cfg.audio_dim,
                                             cfg.dtype, cfg.top_k, p, raster=raster)
    blocked, raster = mk(False), mk(True)
    Ob = blocked.forward(x["Q"], x["K"], x["V"], x["hhat"])
    gb = blocked.backward(x["dO"])
    Or = raster.forward(x["Q"], x["K"], x["V"], x["hhat"])
    gr = raster.backward(x["dO"])
    torch.cuda.synchronize()
    assert raster.status() == 0
    assert torch.equal(Or, Ob)
    assert torch.equal(raster.lse, blocked.lse) and torch.equal(raster.Of32, blocked.Of32)
    for name_, a, b in zip(("dQ", "dK", "dV"), gr, gb):
        assert torch.equal(a, b), name_
    # and the oracle's gradients under the layer's own selection
    nb = raster.num_blocks()
    bs = raster.blk_start[: nb + 1].cpu().numpy().astype(np.int64)
    perm = raster.perm.cpu().numpy().astype(np.int64)
    Qb, Kb, Vb, dOb = (orc.permute(host(x[k]), perm) for k in ("Q", "K", "V", "dO"))
    refs = orc.sparse_attention_bwd(Qb, Kb, Vb, dOb, bs, unpack_sel(raster.sel, nb))
    for a, r in zip(gr, refs):
        assert rel_l2(host(a), orc.unpermute(r, perm)) <= REL_L2[cfg.dtype]


def test_raster_training_full_2k_grid():
    cfg = get_config("2k")
    x = inputs.make_inputs(cfg, "cuda")
    mk = lambda raster: PrismSparseAttention(cfg.T, cfg.H, cfg.W, cfg.heads, cfg.head_dim, cfg.audio_dim,
                                             cfg.dtype, cfg.top_k, cfg.top_p, raster=raster)
    blocked = mk(False)
    Ob = blocked.forward(x["Q"], x["K"], x["V"], x["hhat"])
    gb = blocked.backward(x["dO"])
    torch.cuda.synchronize()
    del blocked
    raster = mk(True)
    Or = raster.forward(x["Q"], x["K"], x["V"], x["hhat"])
    gr = raster.backward(x["dO"])
    torch.cuda.synchronize()
    assert raster.status() == 0
    assert torch.equal(Or, Ob)
    for name_, a, b in zip(("dQ", "dK", "dV"), gr, gb):
        assert torch.equal(a, b), name_
