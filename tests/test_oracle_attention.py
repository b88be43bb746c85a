"""Pins of the oracle's sparse attention (forward and backward) against a
textbook triple loop, torch fp64 autograd, central finite differences and the
dense special case (no GPU)."""
import math

import numpy as np
import pytest
import torch

import oracle as orc


def _case(seed, nb=5, bsz=(2, 4, 3, 1, 2), h=2, d=3):
    rng = np.random.default_rng(seed)
    bs = np.concatenate([[0], np.cumsum(bsz)]).astype(np.int64)
    N = int(bs[-1])
    Q, K, V, dO = (rng.normal(size=(h, N, d)) for _ in range(4))
    sel = rng.uniform(size=(h, nb, nb)) < 0.5
    sel[..., 0] |= ~sel.any(-1)                      # at least one block per row
    return Q, K, V, dO, bs, sel


def _mask(sel, bs):
    h, nb, _ = sel.shape
    N = int(bs[-1])
    m = np.zeros((h, N, N), dtype=bool)
    for hh in range(h):
        for i in range(nb):
            for j in range(nb):
                if sel[hh, i, j]:
                    m[hh, bs[i]:bs[i + 1], bs[j]:bs[j + 1]] = True
    return m


def test_fwd_textbook_triple_loop():
    Q, K, V, _, bs, sel = _case(0)
    O, lse = orc.sparse_attention_fwd(Q, K, V, bs, sel)
    m = _mask(sel, bs)
    h, N, d = Q.shape
    sc = 1 / math.sqrt(d)
    for hh in range(h):
        for q in range(N):
            w = [math.exp(sc * sum(Q[hh, q, c] * K[hh, k, c] for c in range(d))) if m[hh, q, k] else 0.0
                 for k in range(N)]
            z = sum(w)
            for c in range(d):
                assert abs(O[0 if False else hh, q, c] - sum(w[k] * V[hh, k, c] for k in range(N)) / z) < 1e-12
            assert abs(lse[hh, q] - math.log(z)) < 1e-12


def _torch_masked(Q, K, V, m):
    d = Q.shape[-1]
    s = torch.einsum("hqd,hkd->hqk", Q, K) / math.sqrt(d)
    s = s.masked_fill(~torch.from_numpy(m), float("-inf"))
    return torch.softmax(s, -1) @ V


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_fwd_bwd_vs_torch_autograd(seed):
    Q, K, V, dO, bs, sel = _case(seed)
    O, _ = orc.sparse_attention_fwd(Q, K, V, bs, sel)
    dQ, dK, dV = orc.sparse_attention_bwd(Q, K, V, dO, bs, sel)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (Q, K, V))
    to = _torch_masked(tq, tk, tv, _mask(sel, bs))
    to.backward(torch.tensor(dO))
    np.testing.assert_allclose(O, to.detach().numpy(), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(dQ, tq.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dK, tk.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dV, tv.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_bwd_central_finite_differences():
    Q, K, V, dO, bs, sel = _case(4, h=1, d=2)
    dQ, dK, dV = orc.sparse_attention_bwd(Q, K, V, dO, bs, sel)
    L = lambda q, k, v: float((orc.sparse_attention_fwd(q, k, v, bs, sel)[0] * dO).sum())
    eps = 1e-6
    rng = np.random.default_rng(0)
    for X, G, which in ((Q, dQ, 0), (K, dK, 1), (V, dV, 2)):
        for _ in range(6):
            idx = (0, int(rng.integers(X.shape[1])), int(rng.integers(X.shape[2])))
            args_p = [Q.copy(), K.copy(), V.copy()]
            args_m = [Q.copy(), K.copy(), V.copy()]
            args_p[which][idx] += eps
            args_m[which][idx] -= eps
            fd = (L(*args_p) - L(*args_m)) / (2 * eps)
            assert abs(fd - G[idx]) < 1e-7 * max(1.0, abs(fd)), (which, idx, fd, G[idx])


def test_dense_limit_equals_full_softmax_attention():
    # p >= 1 (or k >= n_blk) selects every block -> plain dense softmax attention
    Q, K, V, dO, bs, _ = _case(5)
    nb = len(bs) - 1
    Pfake = np.random.default_rng(0).dirichlet(np.ones(nb), size=(2, nb))
    for k, p in ((1, 1.0), (nb, 0.3)):
        sel = orc.block_select(Pfake, k, p)["sel"]
        assert sel.all()
        O, lse = orc.sparse_attention_fwd(Q, K, V, bs, sel)
        s = np.einsum("hqd,hkd->hqk", Q, K) / math.sqrt(Q.shape[-1])
        ref = torch.softmax(torch.tensor(s), -1).numpy() @ V
        np.testing.assert_allclose(O, ref, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(lse, torch.logsumexp(torch.tensor(s), -1).numpy(), rtol=1e-13)


def test_sampled_equals_full():
    Q, K, V, dO, bs, sel = _case(6)
    O, lse = orc.sparse_attention_fwd(Q, K, V, bs, sel)
    Os, lses = orc.sparse_attention_fwd(Q, K, V, bs, sel, heads=[1], q_blocks=[0, 3])
    for i in (0, 3):
        np.testing.assert_array_equal(Os[0, bs[i]:bs[i + 1]], O[1, bs[i]:bs[i + 1]])
    dQ, dK, dV = orc.sparse_attention_bwd(Q, K, V, dO, bs, sel)
    sq, sk, sv = orc.sparse_attention_bwd(Q, K, V, dO, bs, sel, heads=[1], q_blocks=[2], k_blocks=[1, 4])
    np.testing.assert_allclose(sq[0, bs[2]:bs[3]], dQ[1, bs[2]:bs[3]], rtol=1e-13)
    for j in (1, 4):
        np.testing.assert_allclose(sk[0, bs[j]:bs[j + 1]], dK[1, bs[j]:bs[j + 1]], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(sv[0, bs[j]:bs[j + 1]], dV[1, bs[j]:bs[j + 1]], rtol=1e-12, atol=1e-14)
    assert np.isnan(sk[0, bs[0]:bs[1]]).all()


def test_key_block_gradients_from_known_lse_and_o():
    # teacher-forced dK, dV of sampled key blocks equal the full backward (itself pinned
    # against torch autograd and finite differences) when given the forward's LSE and O
    Q, K, V, dO, bs, sel = _case(8)
    O, lse = orc.sparse_attention_fwd(Q, K, V, bs, sel)
    dQ, dK, dV = orc.sparse_attention_bwd(Q, K, V, dO, bs, sel)
    sk, sv = orc.sparse_attention_bwd_keys(Q, K, V, dO, bs, sel, lse[[1]], O[[1]], heads=[1], k_blocks=[0, 2, 4])
    for j in (0, 2, 4):
        np.testing.assert_allclose(sk[0, bs[j]:bs[j + 1]], dK[1, bs[j]:bs[j + 1]], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(sv[0, bs[j]:bs[j + 1]], dV[1, bs[j]:bs[j + 1]], rtol=1e-12, atol=1e-14)
    assert np.isnan(sk[0, bs[1]:bs[2]]).all()


def test_unselected_keys_get_zero_gradient():
    Q, K, V, dO, bs, sel = _case(7)
    sel[:, :, 2] = False                                  # nobody attends key block 2
    _, dK, dV = orc.sparse_attention_bwd(Q, K, V, dO, bs, sel)
    assert (dK[:, bs[2]:bs[3]] == 0).all() and (dV[:, bs[2]:bs[3]] == 0).all()


def test_run_layer_tiny_end_to_end_invariants():
    from dynamic_block_sparse_macro_b200 import inputs
    from dynamic_block_sparse_macro_b200.configs import get_config
    cfg = get_config("tiny")
    x = inputs.make_inputs(cfg, "cpu")
    f = {k: inputs.to_f64(v) for k, v in x.items()}
    out = orc.run_layer(f["Q"], f["K"], f["V"], f["hhat"], cfg.T, cfg.H, cfg.W,
                        cfg.top_k, cfg.top_p, dO=f["dO"])
    nb = len(out["blk_start"]) - 1
    assert 8 <= nb <= 32
    assert (out["select"]["count"] >= min(cfg.top_k, nb)).all()
    assert np.isfinite(out["O"]).all() and np.isfinite(out["dQ"]).all()
    # dense limit end to end (p = 1): raster output equals full softmax attention
    dense = orc.run_layer(f["Q"], f["K"], f["V"], f["hhat"], cfg.T, cfg.H, cfg.W, 1, 1.0)
    q, k, v = (torch.tensor(f[n]).transpose(0, 1) for n in "QKV")
    ref = torch.softmax(q @ k.transpose(1, 2) / math.sqrt(cfg.head_dim), -1) @ v
    np.testing.assert_allclose(dense["O"], ref.transpose(0, 1).numpy(), rtol=1e-10, atol=1e-12)
