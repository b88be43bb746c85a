"""The dS handoff backward (prism_sparse_attn_bwd_ds and its raster form) on the GPU.

The handoff changes only how dQ is formed. With it, dQ = scale * dS K, where dS is
the blocks that the key-stationary kernel stored. Without it, dQ is formed from
S and dP recomputed. The checks:
  - dK and dV equal the recomputing call's bit for bit;
  - dQ meets the oracle at the bf16 bar, whole-tensor and per (head, block);
  - a buffer too small for the selection leaves the gate off, and the call then
    gives the recomputing call's dQ bit for bit.
The grid of several split tiles is opt-in (PRISM_TEST_DS=1) until it has run on
a B200; the 2K layer's split tiles gave dQ, dK and dV bit-identical to the
recomputing call.
"""
import os

import numpy as np
import pytest
import torch

from dynamic_block_sparse_macro_b200 import _abi, inputs
from dynamic_block_sparse_macro_b200.configs import get_config

pytestmark = pytest.mark.gpu

CASES = {
    "tiny_grid": dict(T=8, H=16, W=16, heads=2),
    "aniso_split_tiles": dict(T=16, H=32, W=32, heads=3),
}
_OPT_IN = pytest.mark.skipif(os.environ.get("PRISM_TEST_DS") != "1", reason="set PRISM_TEST_DS=1")
NAMES = [pytest.param("tiny_grid"), pytest.param("aniso_split_tiles", marks=_OPT_IN)]


def _run(name, d):
    from gpu_parity import run_gpu
    cfg = get_config("720p", head_dim=d, **CASES[name])
    x = inputs.make_inputs(cfg, "cuda")
    mod, O, grads = run_gpu(cfg, x)
    return cfg, x, mod, grads


def _ds_buffer(mod, pieces):
    n = _abi.prism_attn_bwd_ds_bytes(mod.prob, pieces)
    return torch.empty(n, dtype=torch.uint8, device="cuda")


def _pairs(mod, cfg):
    from gpu_parity import unpack_sel
    return int(unpack_sel(mod.gsel, cfg.n_tokens // 64).sum())


@pytest.mark.parametrize("d", [128, 64])
@pytest.mark.parametrize("name", NAMES)
def test_blocked_handoff(name, d):
    import oracle as orc
    from gpu_parity import REL_L2, bits, block_rel_l2, host, rel_l2, unpack_sel
    cfg, x, mod, _ = _run(name, d)
    ds = _ds_buffer(mod, max(1, _pairs(mod, cfg)))
    dQ, dK, dV = (torch.empty_like(mod.dQp) for _ in range(3))
    _abi.prism_sparse_attn_bwd_ds(mod.prob, mod.Qp, mod.Kp, mod.Vp, mod.Op, mod.Of32, mod.dOp, mod.lse, mod.gsel,
                                  mod.gselT, mod.scale, dQ, dK, dV, mod.dev_status, mod.ws_bwd, ds)
    torch.cuda.synchronize()
    assert mod.status() == 0
    assert int(ds[:4].view(torch.int32).item()) == 1          # the gate: every piece fitted
    assert np.array_equal(bits(dK), bits(mod.dKp))
    assert np.array_equal(bits(dV), bits(mod.dVp))
    nb = mod.num_blocks()
    perm, bs = orc.build_permutation(mod.shape_id.cpu().numpy().astype(np.int64), cfg.T, cfg.H, cfg.W)
    sel = unpack_sel(mod.sel, nb)
    Qb, Kb, Vb, dOb = host(mod.Qp), host(mod.Kp), host(mod.Vp), host(mod.dOp)
    dQ_ref, _, _ = orc.sparse_attention_bwd(Qb, Kb, Vb, dOb, bs, sel)
    tol = REL_L2[cfg.dtype]
    got = host(dQ)
    assert rel_l2(got, dQ_ref) <= tol
    assert block_rel_l2(got, dQ_ref, bs, floor=0.1) <= 5 * tol
    # the recomputing call's dQ is within rounding of the handoff's
    assert rel_l2(got, host(mod.dQp)) <= 2e-3


@pytest.mark.parametrize("name", NAMES)
def test_blocked_handoff_too_small_falls_back(name):
    from gpu_parity import bits
    cfg, x, mod, _ = _run(name, 128)
    ds = _ds_buffer(mod, 1)                                   # room for one piece only
    dQ, dK, dV = (torch.empty_like(mod.dQp) for _ in range(3))
    _abi.prism_sparse_attn_bwd_ds(mod.prob, mod.Qp, mod.Kp, mod.Vp, mod.Op, mod.Of32, mod.dOp, mod.lse, mod.gsel,
                                  mod.gselT, mod.scale, dQ, dK, dV, mod.dev_status, mod.ws_bwd, ds)
    torch.cuda.synchronize()
    assert mod.status() == 0
    assert int(ds[:4].view(torch.int32).item()) == 0
    for a, b in ((dQ, mod.dQp), (dK, mod.dKp), (dV, mod.dVp)):
        assert np.array_equal(bits(a), bits(b))


@pytest.mark.parametrize("name", NAMES)
def test_raster_handoff(name):
    from gpu_parity import bits, host, rel_l2
    cfg, x, mod, grads = _run(name, 128)
    ds = _ds_buffer(mod, max(1, _pairs(mod, cfg)))
    dQ, dK, dV = (torch.empty_like(x["Q"]) for _ in range(3))
    _abi.prism_sparse_attn_bwd_raster_ds(mod.prob, x["Q"], x["K"], x["V"], mod.Of32, x["dO"], mod.lse, mod.perm,
                                         mod.shape_id, mod.gsel, mod.gselT, mod.scale, dQ, dK, dV, mod.dev_status,
                                         mod.ws_bwd, ds)
    torch.cuda.synchronize()
    assert mod.status() == 0
    assert int(ds[:4].view(torch.int32).item()) == 1
    # raster results are the blocked results unpermuted, so dK, dV equal the layer's
    assert np.array_equal(bits(dK), bits(grads[1]))
    assert np.array_equal(bits(dV), bits(grads[2]))
    assert rel_l2(host(dQ), host(grads[0])) <= 2e-3
