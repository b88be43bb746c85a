"""GPU vs oracle, every stage, through the C ABI (needs a B200)."""
import numpy as np
import pytest
import torch

from dynamic_block_sparse_macro_b200 import inputs
from dynamic_block_sparse_macro_b200.configs import get_config

pytestmark = pytest.mark.gpu


def _inputs(cfg):
    return inputs.make_inputs(cfg, "cuda")


def test_tiny_f32_all_stages():
    from gpu_parity import check_layer
    cfg = get_config("tiny")
    rep = check_layer(cfg, _inputs(cfg))
    print("tiny", rep)


@pytest.mark.parametrize("d", [128, 64])
def test_bf16_tiny_grid(d):
    # 8x16x16 grid, 2 heads: 16 query tiles per head
    from gpu_parity import check_layer
    cfg = get_config("720p", T=8, H=16, W=16, heads=2, head_dim=d)
    rep = check_layer(cfg, _inputs(cfg))
    print("bf16 tiny", d, rep)


@pytest.mark.parametrize("d", [128, 64])
def test_bf16_aniso_several_tiles(d):
    # 16x32x32 grid (16,384 tokens, 32 zones), 3 heads: mixed block volumes,
    # many 64-row tiles, several selected blocks per row
    from gpu_parity import check_layer
    cfg = get_config("720p", T=16, H=32, W=32, heads=3, head_dim=d)
    rep = check_layer(cfg, _inputs(cfg))
    print("bf16 aniso", d, rep)


def test_f32_fgbg_d128():
    from gpu_parity import check_layer
    cfg = get_config("2k", T=16, H=16, W=32, heads=2, dtype="f32")
    rep = check_layer(cfg, _inputs(cfg))
    assert rep["volume_mix"][256] > 0 and rep["volume_mix"][64] > 0
    print("f32 fgbg", rep)


def test_bf16_fgbg_with_blobs():
    from gpu_parity import check_layer
    cfg = get_config("2k", T=16, H=24, W=32, heads=2)
    rep = check_layer(cfg, _inputs(cfg))
    print("bf16 fgbg", rep)


@pytest.mark.parametrize("top_k,top_p", [(1, 1.0), (10_000, 0.5)])
def test_dense_limit(top_k, top_p):
    # p = 1 or k >= n_blk selects every block: dense attention
    from gpu_parity import check_layer
    cfg = get_config("tiny")
    rep = check_layer(cfg, _inputs(cfg), top_k=top_k, top_p=top_p)
    assert rep["density"] == 1.0


def test_top_k_only():
    from gpu_parity import check_layer
    cfg = get_config("tiny", heads=1)
    rep = check_layer(cfg, _inputs(cfg), top_k=2, top_p=1e-6)
    assert rep["density"] > 0


@pytest.mark.parametrize("guidance", ["video", "audio"])
def test_single_guidance_ablation(guidance):
    # the pages' ablations of the dual guidance: g and rho from one term only
    from gpu_parity import check_layer
    cfg = get_config("tiny")
    check_layer(cfg, _inputs(cfg), guidance=guidance)


@pytest.mark.parametrize("fixed_shape", [3, 10, 14])
def test_fixed_shape_baseline(fixed_shape):
    # the fixed-shape block-sparse baseline: one candidate (64, 128 or 256 tokens) everywhere
    from gpu_parity import check_layer
    cfg = get_config("tiny")
    rep = check_layer(cfg, _inputs(cfg), fixed_shape=fixed_shape)
    vol = {3: 64, 10: 128, 14: 256}[fixed_shape]
    assert rep["volume_mix"][vol] == cfg.n_tokens // 512


def test_top_p_only():
    from gpu_parity import check_layer
    cfg = get_config("tiny", heads=1)
    rep = check_layer(cfg, _inputs(cfg), top_k=0, top_p=0.5)
    assert rep["density"] > 0


def test_degenerate_constant_video_silent_audio():
    # constant V and hhat = 0: zero variances -> r = 1/3, abar = 0, rho = 0 -> B = 256 everywhere
    from gpu_parity import check_layer
    cfg = get_config("tiny")
    x = _inputs(cfg)
    x["V"] = torch.full_like(x["V"], 0.5)
    x["hhat"] = torch.zeros_like(x["hhat"])
    # exact gradients are 0 here (dP - Delta = 0): measure fp32 noise against ||dO||
    rep = check_layer(cfg, x, grad_floor=1.0)
    assert rep["volume_mix"] == {64: 0, 128: 0, 256: 4}


def test_single_zone_grid():
    from gpu_parity import check_layer
    cfg = get_config("tiny", T=8, H=8, W=8, heads=1)
    check_layer(cfg, _inputs(cfg))


def test_deterministic_repeat():
    from gpu_parity import run_gpu
    cfg = get_config("720p", T=8, H=16, W=32, heads=2)
    x = _inputs(cfg)
    m1, O1, g1 = run_gpu(cfg, x)
    O1, g1 = O1.clone(), [t.clone() for t in g1]
    m2, O2, g2 = run_gpu(cfg, x)
    assert torch.equal(O1, O2)
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_inference_layer_matches_training_forward(dtype):
    # with_backward=False: no LSE, no fp32 O, no key-major selection; O and every decision
    # are the bits of the training layer's forward, and O matches the oracle's attention
    # under the inference layer's own selection
    import oracle as orc
    from dynamic_block_sparse_macro_b200.layer import PrismSparseAttention
    from gpu_parity import REL_L2, block_rel_l2, host, rel_l2, run_gpu, unpack_sel
    cfg = get_config("720p", T=16, H=32, W=32, heads=3, dtype=dtype)
    x = _inputs(cfg)
    mt, Ot, _ = run_gpu(cfg, x, backward=False)
    mi = PrismSparseAttention(cfg.T, cfg.H, cfg.W, cfg.heads, cfg.head_dim, cfg.audio_dim, cfg.dtype,
                              cfg.top_k, cfg.top_p, with_backward=False)
    Oi = mi.forward(x["Q"], x["K"], x["V"], x["hhat"])
    torch.cuda.synchronize()
    assert mi.status() == 0 and mi.lse is None
    assert torch.equal(mi.perm, mt.perm) and torch.equal(mi.gsel, mt.gsel)
    assert torch.equal(Oi, Ot)
    nb = mi.num_blocks()
    bs = mi.blk_start[: nb + 1].cpu().numpy().astype(np.int64)
    O_ref, _ = orc.sparse_attention_fwd(host(mi.Qp), host(mi.Kp), host(mi.Vp), bs, unpack_sel(mi.sel, nb))
    Ob = host(mi.Op)
    tol = REL_L2[dtype]
    assert rel_l2(Ob, O_ref) <= tol and block_rel_l2(Ob, O_ref, bs) <= 2 * tol
    perm = mi.perm.cpu().numpy().astype(np.int64)
    np.testing.assert_array_equal(host(Oi), orc.unpermute(Ob, perm))
