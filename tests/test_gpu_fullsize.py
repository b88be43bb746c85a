"""Full-size parity: the 720p, 1080p and 2K layers run exactly as the benchmark
runs them (same configuration, same calls).  What the oracle can do in full is
checked in full (the shapes of every zone, the permutation, the block table);
the rest on samples the oracle computes one by one: raw statistics of sampled
zones (each zone on its own), the grid-wide normalisation from the GPU's own
statistics, bit-exact permuted rows, P rows, O / LSE of sampled query blocks,
dQ of sampled query blocks and dK / dV of sampled key blocks on one sampled
head (the samples always include the query block with the most selected blocks
and the key block most query blocks selected: the split tiles), and every
selection row of every head (two heads at the long grid), all under the GPU's
own upstream decisions."""
import numpy as np
import pytest
import torch

import oracle as orc
from dynamic_block_sparse_macro_b200 import inputs
from dynamic_block_sparse_macro_b200.configs import get_config
from dynamic_block_sparse_macro_b200.layer import PrismSparseAttention

from gpu_parity import NEAR_TIE, REL_L2, rel_l2, unpack_sel

pytestmark = pytest.mark.gpu


def _ratio(s):
    tot = s.sum(axis=-1, keepdims=True)
    return np.where(tot > 0, s / np.where(tot > 0, tot, 1.0), 1.0 / 3.0)


def _f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("name,fixed", [("720p", -1), ("1080p", -1), ("2k", -1), ("2k", 3), ("long", -1)])
def test_full_size_sampled(name, fixed):
    # ("2k", 3): the fixed-shape baseline with 64-token blocks everywhere, 4608 blocks a row,
    # which takes the one-CTA-per-row selection (rows of more than 4096 blocks).
    # "long": 1,032,192 tokens, the first grid whose element offsets pass 2^31.
    cfg = get_config(name)
    T, H, W = cfg.T, cfg.H, cfg.W
    N, Z = cfg.n_tokens, cfg.n_tokens // 512
    dev = torch.device("cuda")
    x = inputs.make_inputs(cfg, "cuda")
    mod = PrismSparseAttention(T, H, W, cfg.heads, cfg.head_dim, cfg.audio_dim, cfg.dtype, cfg.top_k, cfg.top_p,
                               fixed_shape=fixed)
    O = mod.forward(x["Q"], x["K"], x["V"], x["hhat"])
    grads = mod.backward(x["dO"])
    torch.cuda.synchronize()
    assert mod.status() == 0
    rng = np.random.default_rng(11)

    # stage 1: raw statistics of sampled zones, each zone as an 8x8x8 grid of its own
    zs = mod.zone_stats.cpu().double().numpy()
    ZH, ZW = H // 8, W // 8
    for m in rng.choice(Z, 4, replace=False):
        zt, zh, zw = m // (ZH * ZW), (m // ZW) % ZH, m % ZW
        t, h, w = np.meshgrid(np.arange(8) + 8 * zt, np.arange(8) + 8 * zh, np.arange(8) + 8 * zw, indexing="ij")
        rows = torch.as_tensor(((t * H + h) * W + w).reshape(-1), device=dev)
        ind = orc.zone_indicator(_f64(x["V"][rows]), _f64(x["hhat"][rows]), 8, 8, 8)
        np.testing.assert_allclose(zs[m, :3], ind["sigma2_v"][0], rtol=1e-4, atol=1e-7)
        np.testing.assert_allclose(zs[m, 3], ind["rho_raw"][0], rtol=1e-4, atol=1e-7)
        np.testing.assert_allclose(zs[m, 4], ind["A"][0], rtol=1e-5, atol=1e-6)
        np.testing.assert_allclose(zs[m, 5:8], ind["sigma2_a"][0], rtol=1e-4, atol=1e-6)
    # the grid-wide normalisation, from the GPU's statistics of every zone
    g, rho, abar = (mod.g.cpu().double().numpy(), mod.rho.cpu().double().numpy(), mod.abar.cpu().double().numpy())
    A = zs[:, 4]
    ab = A / A.max() if A.max() > 0 else np.zeros_like(A)
    np.testing.assert_allclose(abar, ab, rtol=1e-5, atol=1e-7)
    np.testing.assert_allclose(g, _ratio(zs[:, :3]) + ab[:, None] * _ratio(zs[:, 5:8]) + orc.EPS, rtol=2e-5,
                               atol=1e-6)
    rv = zs[:, 3] / zs[:, 3].max()
    np.testing.assert_allclose(rho, np.maximum(rv, ab), rtol=2e-5, atol=1e-6)

    # stage 2: every zone's shape (teacher-forced), the permutation and the block table bit-exact
    sid = mod.shape_id.cpu().numpy().astype(np.int64)
    if fixed >= 0:
        assert (sid == fixed).all()
    else:
        tf = orc.assign_shapes(g, rho)
        margin = np.minimum(tf["margin_shape"], tf["margin_volume"])
        bad = sid != tf["shape_id"]
        assert (margin[bad] < NEAR_TIE).all()
    perm, bs = orc.build_permutation(sid, T, H, W)
    nb = mod.num_blocks()
    assert nb == len(bs) - 1
    assert np.array_equal(mod.perm.cpu().numpy(), perm)
    assert np.array_equal(mod.blk_start.cpu().numpy()[: nb + 1], bs)

    # stage 3 on one sampled head: the permuted copies are bit copies
    hh = int(rng.integers(cfg.heads))
    perm_t = torch.as_tensor(perm, device=dev, dtype=torch.long)
    for src, dst in (("Q", mod.Qp), ("K", mod.Kp), ("V", mod.Vp)):
        assert torch.equal(dst[hh], x[src][perm_t, hh]), src
    Qh, Kh, Vh = (_f64(t[hh])[None] for t in (mod.Qp, mod.Kp, mod.Vp))

    # stage 4: P rows of sampled query blocks (the oracle pools every block of the head)
    _, _, P = orc.block_pool_score(Qh, Kh, bs, heads=[0])
    Pg = mod.P_view()[hh].cpu().double().numpy()
    sel_g = unpack_sel(mod.sel[hh:hh + 1], nb)[0]
    # the heaviest rows are the split tiles the combine kernels merge: always sampled
    q_heavy = int(sel_g.sum(1).argmax())
    k_heavy = int(sel_g.sum(0).argmax())
    qsamp = sorted(set(rng.choice(nb, 4, replace=False).tolist()) | {q_heavy})
    np.testing.assert_allclose(Pg[qsamp], P[0][qsamp], rtol=1e-4, atol=1e-7)

    # stage 5: every selection row, teacher-forced on the GPU's own P (every head; two at the
    # long grid, whose P holds 4 GB), mismatches only where the oracle's margin is below NEAR_TIE
    heads_sel = range(cfg.heads) if name != "long" else sorted({hh, (hh + cfg.heads // 2) % cfg.heads})
    ties = rows = 0
    for h in heads_sel:
        Ph = mod.P_view()[h].cpu().double().numpy()
        sh = unpack_sel(mod.sel[h:h + 1], nb)[0]
        tsel = orc.block_select(Ph, cfg.top_k, cfg.top_p)
        badr = (sh != tsel["sel"]).any(-1)
        assert (tsel["margin"][badr] < NEAR_TIE).all(), (h, np.nonzero(badr), tsel["margin"][badr])
        ties += int(badr.sum())
        rows += nb
    print(f"{name}: selection near-ties {ties} of {rows} rows ({len(heads_sel)} heads); "
          f"heaviest query block {q_heavy} ({int(sel_g[q_heavy].sum())} blocks), "
          f"key block {k_heavy} selected by {int(sel_g[:, k_heavy].sum())}")

    # stage 6: O and LSE of sampled query blocks under the GPU's selection
    tol = REL_L2[cfg.dtype]
    O_ref, lse_ref = orc.sparse_attention_fwd(Qh, Kh, Vh, bs, sel_g[None], heads=[0], q_blocks=qsamp)
    Ob = _f64(mod.Op[hh])
    lse = mod.lse[hh].cpu().double().numpy()
    for i in qsamp:
        r0, r1 = bs[i], bs[i + 1]
        assert rel_l2(Ob[r0:r1], O_ref[0, r0:r1]) <= tol, i
        assert rel_l2(lse[r0:r1], lse_ref[0, r0:r1]) <= min(tol, 1e-4), i
    # the unpermuted output holds the same bits
    assert torch.equal(O[perm_t, hh], mod.Op[hh])

    # stage 7: dQ of the sampled query blocks, dK / dV of sampled key blocks
    dOh = _f64(x["dO"][perm_t, hh])[None]
    ksamp = sorted(set(rng.choice(nb, 2, replace=False).tolist()) | {k_heavy})
    dQ_ref, _, _ = orc.sparse_attention_bwd(Qh, Kh, Vh, dOh, bs, sel_g[None], heads=[0], q_blocks=qsamp)
    # dK, dV of the sampled key blocks visit every query row that selected them: teacher-forced on
    # the forward's LSE and fp32 O (both checked on samples above) instead of re-normalising each row
    Of = _f64(mod.Of32[hh])[None] if mod.Of32 is not None else Ob[None]
    dK_ref, dV_ref = orc.sparse_attention_bwd_keys(Qh, Kh, Vh, dOh, bs, sel_g[None], lse[None], Of, heads=[0],
                                                   k_blocks=ksamp)
    # per block, as on the small grids: a block's gradient is a cancelling sum (each row of
    # dS sums to zero), so it is measured against at least a tenth of the sampled blocks' RMS
    # norm, at five times the whole-tensor bar
    for dst, ref, blocks in ((mod.dQp, dQ_ref, qsamp), (mod.dKp, dK_ref, ksamp), (mod.dVp, dV_ref, ksamp)):
        got = _f64(dst[hh])
        norms = [float(np.linalg.norm(ref[0, bs[i]:bs[i + 1]])) for i in blocks]
        rms = float(np.sqrt(np.mean(np.square(norms))))
        for i in blocks:
            r0, r1 = bs[i], bs[i + 1]
            assert rel_l2(got[r0:r1], ref[0, r0:r1], 0.1 * rms) <= 5 * tol, i
    for dst, out in zip((mod.dQp, mod.dKp, mod.dVp), grads):
        assert torch.equal(out[perm_t, hh], dst[hh])
