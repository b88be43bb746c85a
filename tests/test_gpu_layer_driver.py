"""The layer object of the C ABI (prism_layer_*): a plain C program
(prism_layer_driver, built beside the library) runs one step from host buffers
through the C ABI alone, and the binding's host-buffer step runs twice in a row
on three streams.  Both must give the bits of the device-buffer layer (the
same deterministic kernels), whose outputs the parity tests check against the
oracle; the driver's outputs are also checked against the oracle directly."""
import os
import subprocess

import numpy as np
import pytest
import torch

import oracle as orc
from dynamic_block_sparse_macro_b200 import build, inputs
from dynamic_block_sparse_macro_b200.configs import get_config
from dynamic_block_sparse_macro_b200.layer import PrismSparseAttention

from gpu_parity import REL_L2, host, rel_l2, unpack_sel

pytestmark = pytest.mark.gpu

CASES = [("720p", dict(T=8, H=16, W=16, heads=2)), ("tiny", {})]


def _layer(cfg):
    return PrismSparseAttention(cfg.T, cfg.H, cfg.W, cfg.heads, cfg.head_dim, cfg.audio_dim, cfg.dtype,
                                cfg.top_k, cfg.top_p)


def _raw(t):
    return t.detach().contiguous().cpu().view(torch.uint8).numpy()


@pytest.mark.parametrize("name,kw", CASES)
def test_c_driver_step_from_host_buffers(tmp_path, name, kw):
    cfg = get_config(name, **kw)
    x = inputs.make_inputs(cfg, "cuda")
    dt = 1 if cfg.dtype == "bf16" else 0
    (tmp_path / "problem.txt").write_text(
        f"{cfg.T} {cfg.H} {cfg.W} {cfg.heads} {cfg.head_dim} {cfg.audio_dim} {dt} {cfg.top_k} {cfg.top_p!r} 1\n")
    for k in ("Q", "K", "V", "hhat", "dO"):
        _raw(x[k]).tofile(tmp_path / f"{k}.bin")
    drv = build.build_driver()
    r = subprocess.run([drv, "run", str(tmp_path)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr + r.stdout
    assert "dev_status 0" in r.stdout

    mod = _layer(cfg)
    O = mod.forward(x["Q"], x["K"], x["V"], x["hhat"])
    grads = mod.backward(x["dO"])
    torch.cuda.synchronize()
    for k, ref in zip(("O", "dQ", "dK", "dV"), (O,) + tuple(grads)):
        got = np.fromfile(tmp_path / f"{k}.bin", dtype=np.uint8)
        np.testing.assert_array_equal(got, _raw(ref).reshape(-1), err_msg=k)

    # and against the oracle under the layer's own selection
    nb = mod.num_blocks()
    bs = mod.blk_start[: nb + 1].cpu().numpy().astype(np.int64)
    perm = mod.perm.cpu().numpy().astype(np.int64)
    sel = unpack_sel(mod.sel, nb)
    Qb, Kb, Vb = host(mod.Qp), host(mod.Kp), host(mod.Vp)
    O_ref, _ = orc.sparse_attention_fwd(Qb, Kb, Vb, bs, sel)
    g_ref = orc.sparse_attention_bwd(Qb, Kb, Vb, orc.permute(host(x["dO"]), perm), bs, sel)
    tdt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    shape = tuple(x["Q"].shape)
    tol = REL_L2[cfg.dtype]
    for k, ref in zip(("O", "dQ", "dK", "dV"), (O_ref,) + tuple(g_ref)):
        got = torch.from_numpy(np.fromfile(tmp_path / f"{k}.bin", dtype=np.uint8)).view(tdt).reshape(shape)
        assert rel_l2(host(got), orc.unpermute(ref, perm)) <= tol, k


def test_host_step_twice_on_three_streams():
    cfg = get_config("720p", T=16, H=32, W=32, heads=3)
    x = inputs.make_inputs(cfg, "cuda")
    mod = _layer(cfg)
    O = mod.forward(x["Q"], x["K"], x["V"], x["hhat"])
    grads = mod.backward(x["dO"])
    ref = [t.cpu() for t in (O,) + tuple(grads)]
    dev = {k: torch.empty_like(x[k]) for k in ("Q", "K", "V", "hhat", "dO")}
    outs = [torch.empty_like(x["Q"]) for _ in range(4)]
    mod.attach_io(dev["Q"], dev["K"], dev["V"], dev["hhat"], outs[0], dev["dO"], *outs[1:])
    hin = {k: x[k].cpu().pin_memory() for k in ("Q", "K", "V", "hhat", "dO")}
    compute, h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    for step in range(2):
        hout = [torch.empty(x["Q"].shape, dtype=x["Q"].dtype).pin_memory() for _ in range(4)]
        mod.step_host(hin["Q"], hin["K"], hin["V"], hin["hhat"], hin["dO"], *hout, compute, h2d, d2h)
        d2h.synchronize()
        for k, a, b in zip(("O", "dQ", "dK", "dV"), hout, ref):
            assert torch.equal(a, b), (step, k)
    compute.synchronize()
    assert mod.status() == 0


@pytest.mark.parametrize("raster", [False, True])
def test_host_steps_back_to_back_with_different_inputs(raster):
    """Two host-buffer steps issued back to back, with different inputs and no
    synchronisation between them.  The second step's uploads may start as soon as
    the first has read its raster inputs (in the blocked layout, after its
    permutes), so an upload that overwrote an input still being read would change
    the first step's outputs.  Each step must give the device-buffer layer's bits
    for its own inputs."""
    cfg_a = get_config("720p", T=16, H=32, W=32, heads=3)
    cfg_b = get_config("720p", T=16, H=32, W=32, heads=3, seed=cfg_a.seed + 7)
    xs = [inputs.make_inputs(c, "cuda") for c in (cfg_a, cfg_b)]
    mod = PrismSparseAttention(cfg_a.T, cfg_a.H, cfg_a.W, cfg_a.heads, cfg_a.head_dim, cfg_a.audio_dim, cfg_a.dtype,
                               cfg_a.top_k, cfg_a.top_p, raster=raster)
    refs = []
    for x in xs:
        O = mod.forward(x["Q"], x["K"], x["V"], x["hhat"])
        grads = mod.backward(x["dO"])
        torch.cuda.synchronize()
        refs.append([t.cpu() for t in (O,) + tuple(grads)])
    assert not all(torch.equal(a, b) for a, b in zip(*refs))      # the two steps differ
    names = ("Q", "K", "V", "hhat", "dO")
    dev = {k: torch.empty_like(xs[0][k]) for k in names}
    outs = [torch.empty_like(xs[0]["Q"]) for _ in range(4)]
    mod.attach_io(dev["Q"], dev["K"], dev["V"], dev["hhat"], outs[0], dev["dO"], *outs[1:])
    hins = [{k: x[k].cpu().pin_memory() for k in names} for x in xs]
    houts = [[torch.empty(xs[0]["Q"].shape, dtype=xs[0]["Q"].dtype).pin_memory() for _ in range(4)] for _ in xs]
    compute, h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    for rep in range(2):
        for hin, hout in zip(hins, houts):
            mod.step_host(hin["Q"], hin["K"], hin["V"], hin["hhat"], hin["dO"], *hout, compute, h2d, d2h)
        d2h.synchronize()
        for step, (hout, ref) in enumerate(zip(houts, refs)):
            for k, a, b in zip(("O", "dQ", "dK", "dV"), hout, ref):
                assert torch.equal(a, b), (rep, step, k)
    compute.synchronize()
    assert mod.status() == 0
    mod.release()
    assert not mod.L.io_events
