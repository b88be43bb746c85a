"""prism_zone_indicator_noalloc: the zone indicator for callers that cannot
allocate device memory (a C host with no device allocator of its own, or a
service whose device footprint is fixed at start-up).  Its scratch is a
fixed array inside the library; these tests check, through the C ABI, that
it gives the same bits as prism_zone_indicator with a caller-owned
workspace (both run the same deterministic kernels), on calls in a row and on
the largest problem the array holds, and that oversize problems are refused.

This file is named so that pytest collects it last."""
import ctypes
import types

import numpy as np
import pytest
import torch

from dynamic_block_sparse_macro_b200 import _abi, inputs
from dynamic_block_sparse_macro_b200.configs import get_config


def test_oversize_problem_is_refused_before_any_launch():
    from dynamic_block_sparse_macro_b200 import build
    build.build()
    L = _abi.lib()
    # 112x72x128 f32 with 24 heads x 128 needs 3.2 MB of scratch > 2 MiB
    p = _abi.problem(112, 72, 128, 24, 128, 64, "f32")
    fake = 1 << 40                      # never dereferenced: the call must stop at the size check
    assert L.prism_zone_indicator_noalloc(ctypes.byref(p), fake, fake, 1e-6, fake, fake, fake, None,
                                          None) == 4          # PRISM_ERR_WORKSPACE
    # a bad grid is still a shape error
    p = _abi.problem(112, 72, 120 + 4, 24, 128, 64, "bf16")
    assert L.prism_zone_indicator_noalloc(ctypes.byref(p), fake, fake, 1e-6, fake, fake, fake, None,
                                          None) == 2          # PRISM_ERR_SHAPE


def _run(cfg, x, noalloc):
    prob = _abi.problem(cfg.T, cfg.H, cfg.W, cfg.heads, cfg.head_dim, cfg.audio_dim, cfg.dtype)
    sz = _abi.query_sizes(prob)
    Z = sz.n_zones
    out = {k: torch.full(s, float("nan"), device="cuda") for k, s in
           (("g", (Z, 3)), ("rho", (Z,)), ("abar", (Z,)), ("zs", (Z, 8)))}
    if noalloc:
        _abi.prism_zone_indicator_noalloc(prob, x["V"], x["hhat"], 1e-6, out["g"], out["rho"], out["abar"],
                                          out["zs"])
    else:
        ws = torch.empty(sz.ws_indicator, dtype=torch.uint8, device="cuda")
        _abi.prism_zone_indicator(prob, x["V"], x["hhat"], 1e-6, out["g"], out["rho"], out["abar"], out["zs"],
                                  ws)
    torch.cuda.synchronize()
    return {k: v.cpu().numpy() for k, v in out.items()}


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_twice_in_a_row():
    # two different problems back to back: the second call reuses the shared
    # scratch left by the first and must not depend on its contents
    cases = [get_config("2k", T=16, H=24, W=32, heads=4), get_config("tiny")]
    for cfg in cases + cases[:1]:
        x = inputs.make_inputs(cfg, "cuda", with_grad=False)
        ref = _run(cfg, x, noalloc=False)
        got = _run(cfg, x, noalloc=True)
        for k in ref:
            assert np.isfinite(got[k]).all(), k
            np.testing.assert_array_equal(got[k], ref[k], err_msg=k)


@pytest.mark.gpu
def test_noalloc_at_the_scratch_limit():
    # 256^3 tokens (the most a problem may have: 32,768 zones), one bf16 head of 128
    # channels: 32,768 zones x 16 floats = exactly the 2 MiB of the array
    T = H = W = 256
    prob = _abi.problem(T, H, W, 1, 128, 64, "bf16")
    sz = _abi.query_sizes(prob)
    assert sz.ws_indicator == _abi.NOALLOC_SCRATCH_BYTES
    gen = torch.Generator(device="cuda").manual_seed(20261231)
    N = T * H * W
    x = {"V": torch.randn((N, 1, 128), generator=gen, device="cuda", dtype=torch.bfloat16),
         "hhat": torch.randn((N, 64), generator=gen, device="cuda", dtype=torch.bfloat16)}
    cfg = types.SimpleNamespace(T=T, H=H, W=W, heads=1, head_dim=128, audio_dim=64, dtype="bf16")
    for _ in range(2):
        ref = _run(cfg, x, noalloc=False)
        got = _run(cfg, x, noalloc=True)
        for k in ref:
            assert np.isfinite(got[k]).all(), k
            np.testing.assert_array_equal(got[k], ref[k], err_msg=k)
