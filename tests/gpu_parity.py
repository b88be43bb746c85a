"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and compare each stage with the fp64 oracle, teacher-forced (the oracle gets
the GPU's upstream decisions) so that one near-tie does not cascade.

Tolerances (the bar): integer/index outputs bit-exact except decisions whose
oracle margin is below NEAR_TIE (counted and returned); attention outputs
and gradients within relative L2 error 1e-5 (f32 storage) or 1e-2 (bf16)
over the whole tensor, and every (head, block) on its own (O at twice that,
gradients at five times that against at least a tenth of the typical block
norm) so that one bad tile cannot hide among hundreds of good ones."""
from __future__ import annotations

import numpy as np
import torch

import oracle as orc
from dynamic_block_sparse_macro_b200 import inputs
from dynamic_block_sparse_macro_b200.layer import PrismSparseAttention

NEAR_TIE = 1e-5
REL_L2 = {"f32": 1e-5, "bf16": 1e-2}


def rel_l2(a, b, floor=0.0):
    """||a - b|| / max(||b||, floor).  The floor keeps an exactly-zero reference
    (e.g. the gradients of a constant V) from turning fp32 rounding noise into
    an unbounded relative error."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = max(float(np.linalg.norm(b)), floor)
    return float(np.linalg.norm(a - b) / (den if den > 0 else 1.0))


def block_rel_l2(a, b, bs, floor=0.0):
    """Largest relative L2 error over the (head, block) pieces of blocked [h, N, d]
    (or [h, N]) arrays; a block's denominator is at least `floor` times the RMS
    block norm of the reference (0: no floor)."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    nb = len(bs) - 1
    num = np.empty((a.shape[0], nb))
    den = np.empty((a.shape[0], nb))
    for i in range(nb):
        sl = slice(int(bs[i]), int(bs[i + 1]))
        num[:, i] = np.sqrt(((a[:, sl] - b[:, sl]) ** 2).reshape(a.shape[0], -1).sum(-1))
        den[:, i] = np.sqrt((b[:, sl] ** 2).reshape(a.shape[0], -1).sum(-1))
    rms = float(np.sqrt((den ** 2).mean()))
    den = np.maximum(den, floor * rms)
    ok = den > 0
    return float((num[ok] / den[ok]).max()) if ok.any() else float(num.max())


def unpack_sel(words: torch.Tensor, nb: int) -> np.ndarray:
    """[h, MB, SW] int32 bitmask -> bool [h, nb, nb]."""
    w = words[:, :nb, :].contiguous().cpu().numpy().view(np.uint32)
    bits = np.unpackbits(w.view(np.uint8), axis=-1, bitorder="little")
    return bits[..., :nb].astype(bool)


def host(x):
    return inputs.to_f64(x)


def bits(t: torch.Tensor) -> np.ndarray:
    """Raw storage bits of a tensor as a numpy integer array (bit-exact compares)."""
    it = {2: torch.int16, 4: torch.int32}[t.element_size()]
    return t.detach().cpu().contiguous().view(it).numpy()


def run_gpu(cfg, x, top_k=None, top_p=None, backward=True, guidance="joint", fixed_shape=-1):
    mod = PrismSparseAttention(cfg.T, cfg.H, cfg.W, cfg.heads, cfg.head_dim, cfg.audio_dim,
                               cfg.dtype, cfg.top_k if top_k is None else top_k, cfg.top_p if top_p is None else top_p,
                               guidance=guidance, fixed_shape=fixed_shape)
    O = mod.forward(x["Q"], x["K"], x["V"], x["hhat"])
    grads = mod.backward(x["dO"]) if backward else None
    torch.cuda.synchronize()
    return mod, O, grads


def check_layer(cfg, x, top_k=None, top_p=None, backward=True, heads=None, grad_floor=0.0,
                guidance="joint", fixed_shape=-1):
    """Run the GPU layer and check every stage; returns a report dict.

    grad_floor: the gradients' relative errors are taken against at least this
    fraction of ||dO||.  Only a case whose exact gradients are zero needs one
    (fp32 rounding noise against a zero reference); every other case uses 0."""
    top_k = cfg.top_k if top_k is None else top_k
    top_p = cfg.top_p if top_p is None else top_p
    mod, O, grads = run_gpu(cfg, x, top_k, top_p, backward, guidance, fixed_shape)
    rep = {}
    T, H, W = cfg.T, cfg.H, cfg.W
    Vh, hh = host(x["V"]), host(x["hhat"])

    # stage 1: indicator (fp32 on the GPU vs fp64 oracle)
    ind = orc.zone_indicator(Vh, hh, T, H, W, guidance=guidance)
    g, rho, abar = (mod.g.cpu().double().numpy(), mod.rho.cpu().double().numpy(),
                    mod.abar.cpu().double().numpy())
    zs = mod.zone_stats.cpu().double().numpy()
    assert np.allclose(g, ind["g"], rtol=2e-5, atol=1e-6), np.abs(g - ind["g"]).max()
    assert np.allclose(rho, ind["rho"], rtol=2e-5, atol=1e-6), np.abs(rho - ind["rho"]).max()
    assert np.allclose(abar, ind["abar"], rtol=2e-5, atol=1e-6)
    assert np.allclose(zs[:, :3], ind["sigma2_v"], rtol=1e-4, atol=1e-7)
    assert np.allclose(zs[:, 3], ind["rho_raw"], rtol=1e-4, atol=1e-7)
    assert np.allclose(zs[:, 4], ind["A"], rtol=1e-5, atol=1e-6)

    # stage 2: shapes, teacher-forced on the GPU's g / rho, and end to end
    sid = mod.shape_id.cpu().numpy().astype(np.int64)
    if fixed_shape >= 0:                              # the fixed-shape baseline takes no decision
        tf = orc.assign_shapes_fixed(len(sid), fixed_shape)
        assert np.array_equal(sid, tf["shape_id"])
        rep["shape_near_ties"] = 0
    else:
        tf = orc.assign_shapes(g, rho)
        margin = np.minimum(tf["margin_shape"], tf["margin_volume"])
        bad = sid != tf["shape_id"]
        assert (margin[bad] < NEAR_TIE).all(), (np.nonzero(bad), margin[bad])
        e2e = orc.assign_shapes(ind["g"], ind["rho"])
        m2 = np.minimum(e2e["margin_shape"], e2e["margin_volume"])
        bad2 = sid != e2e["shape_id"]
        assert (m2[bad2] < NEAR_TIE).all()
        rep["shape_near_ties"] = int(bad2.sum())
    rep["volume_mix"] = {int(b): int((tf["B"] == b).sum()) for b in (64, 128, 256)}

    # permutation and block table: bit-exact from the GPU's shapes
    perm, bs = orc.build_permutation(sid, T, H, W)
    nb = mod.num_blocks()
    assert nb == len(bs) - 1
    assert np.array_equal(mod.perm.cpu().numpy(), perm)
    gbs = mod.blk_start.cpu().numpy()
    assert np.array_equal(gbs[: nb + 1], bs) and (gbs[nb + 1:] == cfg.n_tokens).all()
    gran = np.repeat(np.arange(nb), np.diff(bs) // 64)
    assert np.array_equal(mod.gran_blk.cpu().numpy(), gran)

    # stage 3: permute is a bit copy
    for name, dev in (("Q", mod.Qp), ("K", mod.Kp), ("V", mod.Vp)):
        assert np.array_equal(bits(dev), orc.permute(bits(x[name]), perm)), name
    Qb, Kb, Vb = host(mod.Qp), host(mod.Kp), host(mod.Vp)

    # stage 4: pooled probabilities
    _, _, P = orc.block_pool_score(Qb, Kb, bs)
    Pg = mod.P_view().cpu().double().numpy()
    assert np.allclose(Pg, P, rtol=1e-4, atol=1e-7), np.abs(Pg - P).max()

    # stage 5: selection, teacher-forced on the GPU's P, then end to end
    sel_g = unpack_sel(mod.sel, nb)
    cnt = mod.sel_count.cpu().numpy()[:, :nb]
    assert np.array_equal(sel_g.sum(-1), cnt)
    tf = orc.block_select(Pg, top_k, top_p)
    badr = (sel_g != tf["sel"]).any(-1)
    assert (tf["margin"][badr] < NEAR_TIE).all(), (badr.sum(), tf["margin"][badr])
    e2e = orc.block_select(P, top_k, top_p)
    badr2 = (sel_g != e2e["sel"]).any(-1)
    assert (e2e["margin"][badr2] < NEAR_TIE).all()
    rep["select_near_ties"] = int(badr2.sum())
    # the kernel's own margin (fp32 sums) against the oracle's on the same P
    mg = mod.margin_sel.cpu().double().numpy()[:, :nb]
    om = tf["margin"]
    fin = np.isfinite(om) & (om > 1e-4)
    assert (np.isinf(mg) == np.isinf(om)).all()
    assert np.allclose(mg[fin], om[fin], rtol=1e-3, atol=2e-6), np.abs(mg[fin] - om[fin]).max()
    rep["density"] = float(sel_g.mean())
    # granule-level view: row qg, bit kg set iff block(kg) in S_block(qg); and its transpose
    G = unpack_sel(mod.gsel, cfg.n_tokens // 64)
    gb = np.repeat(np.arange(nb), np.diff(bs) // 64)
    assert np.array_equal(G, sel_g[:, gb][:, :, gb])
    assert np.array_equal(unpack_sel(mod.gselT, cfg.n_tokens // 64), G.transpose(0, 2, 1))

    # stage 6: attention under the GPU's own selection
    hs = list(range(cfg.heads)) if heads is None else heads
    O_ref, lse_ref = orc.sparse_attention_fwd(Qb, Kb, Vb, bs, sel_g, heads=hs)
    Ob = host(mod.Op)[hs]
    lse = mod.lse.cpu().double().numpy()[hs]
    tol = REL_L2[cfg.dtype]
    rep["O_rel_l2"] = rel_l2(Ob, O_ref)
    rep["lse_rel_l2"] = rel_l2(lse, lse_ref)
    assert rep["O_rel_l2"] <= tol and rep["lse_rel_l2"] <= min(tol, 1e-4), rep
    # the same bar, doubled, on every (head, query block) by itself
    rep["O_block_max_rel_l2"] = block_rel_l2(Ob, O_ref, bs)
    assert rep["O_block_max_rel_l2"] <= 2 * tol, rep
    # unpermute: bit copy back to raster
    assert np.array_equal(bits(O), orc.unpermute(bits(mod.Op), perm))

    if backward:
        dOb = orc.permute(host(x["dO"]), perm)
        dQ_ref, dK_ref, dV_ref = orc.sparse_attention_bwd(Qb, Kb, Vb, dOb, bs, sel_g, heads=hs)
        # gradient scale floor: a fraction (default 1e-4) of ||dO|| over the same heads
        floor = grad_floor * float(np.linalg.norm(dOb[hs]))
        for name, dev, ref in (("dQ", mod.dQp, dQ_ref), ("dK", mod.dKp, dK_ref), ("dV", mod.dVp, dV_ref)):
            got = host(dev)[hs]
            rep[name + "_rel_l2"] = rel_l2(got, ref, floor)
            assert rep[name + "_rel_l2"] <= tol, rep
            # per (head, block).  Every row of dS sums to zero over its keys, so a
            # block's gradient is a cancelling sum that can be much smaller than the
            # terms forming it (and a key block no query selected has an exact zero
            # gradient): blocks are measured against at least 10% of the RMS block
            # norm, at 5x the whole-tensor bar.  A wrong tile still fails by orders
            # of magnitude.
            rep[name + "_block_max_rel_l2"] = block_rel_l2(got, ref, bs, floor=0.1)
            assert grad_floor > 0 or rep[name + "_block_max_rel_l2"] <= 5 * tol, rep
        for dev, out in zip((mod.dQp, mod.dKp, mod.dVp), grads):
            assert np.array_equal(bits(out), orc.unpermute(bits(dev), perm))
    assert mod.status() == 0
    return rep
