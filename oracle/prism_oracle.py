"""Plain fp64 CPU oracle of the Prism dynamic block-sparse video self-attention.

TEST INFRASTRUCTURE ONLY: used by ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline legs of ``bench.py``; never by the product path.  It shares no
code, table or constant generator with the CUDA library.

Source: "Prism: Dynamic Sparse Attention for Native 2K Joint Video-Audio
Generation Model Training" (arXiv 2610.05416), as rendered on three reading
guides and a news page.  Citation keys used below:

  [PT-Ideias]  Portuguese guide (xyznot.com/pt), "Ideias centrais"
  [PT-M1]      Portuguese guide, "Método" 1 "Formulação do Indicador de Variação"
               (equations for sigma^2_{v,d}, r_{v,d}, a, abar, vhat_{a,d}, g_d)
  [PT-M2]      Portuguese guide, "Método" 2 "Volume do Bloco e Quantização do
               Formato" (tau_128, tau_256, B(m), l*_d, s*)
  [PT-M3]      Portuguese guide, "Método" 3 "Atenção Híbrida Top-k / Top-p"
               (pooled K_bar_j, block probabilities P_i, S_i)
  [ZH-FAQ2]    Chinese guide (xyznot.com/zh), FAQ "why macro-zones": blocks are
               multiples of 64 tokens
  [ZH-FAQ4]    Chinese guide, FAQ "how is error propagation avoided": rho, g, P
               are detached; gradients flow only through the sparse attention
  [NEWS-4]     sd114.wiki news page, "工作原理" step 4: sparse kernel over the
               selected blocks, then restore the original spatio-temporal layout

Readings where the pages are silent, garbled or ambiguous:
  R1  D = all heads x head_dim channels of V; one shape per zone, shared by heads.
  R2  rho(m) = max(rho_v(m), abar(m)), rho_v = zone's mean token variance of V
      over channels, divided by its maximum over the zones of the grid.
  R3  abar(m) = A(m) / max_m' A(m'), A(m) = zone mean of a (0 if the max is 0).
  R4  vhat_{a,d} = the r_{v,d} construction applied to the scalar field a.
  R5  eps = 1e-6.
  R6  zero total variance -> ratios 1/3 each.
  R7  rho >= tau_128 -> B=64; tau_256 <= rho < tau_128 -> 128; rho < tau_256 -> 256.
  R8  C_B = power-of-two edges in {2,4,8} with product B: 7 + 6 + 3 = 16 shapes.
  R9  ties in the nearest-shape search (distances equal up to 1e-12) go to the
      lexicographically smallest (b_T, b_H, b_W).
  R10 permutation order: zones in raster order, blocks in raster order inside
      the zone, tokens in raster order inside the block (W fastest everywhere).
  R11 pooling, scores, probabilities and selection are per head.
  R12 s_ij = Qbar_i . Kbar_j / sqrt(d); P_i = softmax_j over all key blocks.
  R13 Top-p = the shortest prefix of the order (P desc, j asc) whose sum is
      >= p; p >= 1 or a sum that never reaches p -> all blocks.
  R14 no forced diagonal block.   R15 non-causal, scale 1/sqrt(d).   R16 batch 1.
  R17 the GPU accumulates stages 1-5 in fp32 from the stored dtype; this oracle
      reads the same stored values in fp64, and decisions are compared outside a
      1e-5 near-tie margin.
  R18 Delta = rowsum(dO * O) uses the unrounded O (an fp32 copy for bf16 storage).
  R19 single-guidance ablations: video only -> g_d = r_{v,d} + eps, rho = rho_v;
      audio only -> g_d = abar * vhat_{a,d} + eps, rho = abar.
  R20 fixed-shape baseline: one candidate shape for every zone, ignoring g, rho
      and tau; the permutation and everything after it are unchanged.
  R21 Top-p only is k = 0; Top-k only is a p so small that the Top-p prefix is
      one block.

Shape ids: the 16 candidates numbered by (volume, b_T, b_H, b_W) ascending.

Layouts: raster token index r = (t*H + h)*W + w.  Raster tensors [N, heads, d];
blocked tensors [heads, N, d] with tokens in permutation order.
"""
from __future__ import annotations

import math
from itertools import product

import numpy as np

ZONE = 8                      # Z_T = Z_H = Z_W = 8            [PT-Ideias], [PT-M1]
TAU_128 = 0.5                 # thresholds on rho(m)           [PT-M2]
TAU_256 = 0.25
EPS = 1e-6                    # R5
VOLUMES = (64, 128, 256)      # B(m)                           [PT-M2], [ZH-FAQ2]
TIE_TOL = 1e-12               # R9

__all__ = [
    "ZONE", "TAU_128", "TAU_256", "EPS", "VOLUMES",
    "candidate_shapes", "zone_indicator", "block_volume", "optimal_log_edges",
    "assign_shapes", "assign_shapes_fixed", "build_permutation", "permute", "unpermute",
    "block_pool_score", "block_select", "sparse_attention_fwd",
    "sparse_attention_bwd", "sparse_attention_bwd_keys", "run_layer",
]


# --------------------------------------------------------------------------
# Candidate shapes (R8): edges in {2, 4, 8}, product B in {64, 128, 256}.
# --------------------------------------------------------------------------
def candidate_shapes():
    """Return (edges [16,3] int, volume [16] int), sorted by (volume, edges)."""
    rows = []
    for B in VOLUMES:
        for e in product((2, 4, 8), repeat=3):
            if e[0] * e[1] * e[2] == B:
                rows.append((B,) + e)
    rows.sort()
    arr = np.array(rows, dtype=np.int64)
    return arr[:, 1:], arr[:, 0]


# --------------------------------------------------------------------------
# Stage 1: zones and the dual-guidance variation indicator        [PT-M1]
# --------------------------------------------------------------------------
def _zones(X, T, H, W):
    """[N, C] raster -> [ZT, ZH, ZW, 8(t), 8(h), 8(w), C]."""
    C = X.shape[-1]
    x = X.reshape(T // ZONE, ZONE, H // ZONE, ZONE, W // ZONE, ZONE, C)
    return x.transpose(0, 2, 4, 1, 3, 5, 6)


def _ratio(s):
    """Normalise three directional variances to sum 1 (R6: 1/3 each if all 0)."""
    tot = s.sum(axis=-1, keepdims=True)
    out = np.full_like(s, 1.0 / 3.0)
    nz = tot[..., 0] > 0
    out[nz] = s[nz] / tot[nz]
    return out


def _directional_variance(Xz):
    """sigma^2_d = (1/C) sum_c (1/Z_d) sum_i (Xbar^{(d)}_{i,c} - mu_c)^2 for d = T, H, W.

    Xz: [..., 8, 8, 8, C].  Xbar^{(d)}_{i,c} is the mean of channel c over the
    other two local axes at position i along axis d; mu_c is the zone mean.
    Returns [..., 3] and mu [..., C].
    """
    mu = Xz.mean(axis=(-4, -3, -2))
    prof = (Xz.mean(axis=(-3, -2)),    # along T: mean over (h, w) -> [..., 8, C]
            Xz.mean(axis=(-4, -2)),    # along H: mean over (t, w)
            Xz.mean(axis=(-4, -3)))    # along W: mean over (t, h)
    sig = [((p - mu[..., None, :]) ** 2).mean(axis=-2).mean(axis=-1) for p in prof]
    return np.stack(sig, axis=-1), mu


def zone_indicator(V, hhat, T, H, W, eps=EPS, guidance="joint"):
    """Per-zone g_d(m), rho(m), abar(m) and the statistics they come from.

    guidance: "joint" (the method), or the single-guidance ablations the
    pages compare against (R19): "video" keeps only the video term of every
    output that combines the two (g_d = r_{v,d} + eps, rho = rho_v), "audio"
    only the audio term (g_d = abar * vhat_{a,d} + eps, rho = abar).

    V: raster [N, D] (or [N, heads, d], flattened to D = heads*d, R1), any float
    dtype (converted to fp64 one temporal slab of zones at a time).
    hhat: raster [N, Da], the cached A2V cross-attention output.

      sigma^2_{v,d}(m), r_{v,d}(m)       [PT-M1] first equation (population variance)
      a = ||hhat||_2, A(m), abar(m)      [PT-M1], R3
      vhat_{a,d}(m)                      R4
      g_d = r_{v,d} + abar * vhat_{a,d} + eps            [PT-M1] second equation
      rho_raw(m) = (1/D) sum_c (1/512) sum_zone (V_c - mu_c)^2,  rho = max(rho_raw/max rho_raw, abar)  R2
    Returns a dict of fp64 arrays with a leading zone axis Z (raster zone order).
    """
    N = T * H * W
    V = np.asarray(V).reshape(N, -1)
    hhat = np.asarray(hhat).reshape(N, -1)
    ZT, ZH, ZW = T // ZONE, H // ZONE, W // ZONE
    slab = ZONE * H * W
    sig_v = np.empty((ZT, ZH, ZW, 3))
    rho_raw = np.empty((ZT, ZH, ZW))
    for zt in range(ZT):
        Vz = _zones(V[zt * slab:(zt + 1) * slab].astype(np.float64), ZONE, H, W)[0]
        s, mu = _directional_variance(Vz)
        sig_v[zt] = s
        rho_raw[zt] = ((Vz - mu[:, :, None, None, None, :]) ** 2).mean(axis=(2, 3, 4)).mean(axis=-1)
    r_v = _ratio(sig_v)

    a = np.sqrt((hhat.astype(np.float64) ** 2).sum(axis=-1))          # a_{t,h,w}
    az = _zones(a[:, None], T, H, W)                                    # [..., 8,8,8,1]
    sig_a, A = _directional_variance(az)
    A = A[..., 0]
    Amax = A.max()
    abar = A / Amax if Amax > 0 else np.zeros_like(A)
    vhat = _ratio(sig_a)

    if guidance not in ("joint", "video", "audio"):
        raise ValueError(guidance)
    use_v = 0.0 if guidance == "audio" else 1.0
    use_a = 0.0 if guidance == "video" else 1.0
    g = use_v * r_v + use_a * abar[..., None] * vhat + eps
    rmax = rho_raw.max()
    rho_v = rho_raw / rmax if rmax > 0 else np.zeros_like(rho_raw)
    rho = np.maximum(use_v * rho_v, use_a * abar)

    Z = ZT * ZH * ZW
    return {
        "g": g.reshape(Z, 3), "rho": rho.reshape(Z), "abar": abar.reshape(Z),
        "r_v": r_v.reshape(Z, 3), "vhat_a": vhat.reshape(Z, 3),
        "sigma2_v": sig_v.reshape(Z, 3), "sigma2_a": sig_a.reshape(Z, 3),
        "rho_raw": rho_raw.reshape(Z), "rho_v": rho_v.reshape(Z), "A": A.reshape(Z),
    }


# --------------------------------------------------------------------------
# Stage 2: block volume and shape quantisation                    [PT-M2]
# --------------------------------------------------------------------------
def block_volume(rho, tau128=TAU_128, tau256=TAU_256):
    """B(m) from rho(m) against tau_128 and tau_256 (R7)."""
    rho = np.asarray(rho, dtype=np.float64)
    return np.where(rho >= tau128, 64, np.where(rho >= tau256, 128, 256)).astype(np.int64)


def optimal_log_edges(g, B):
    """l*_d = -1/2 log2 g_d + (S + 1/2 sum_d' log2 g_d') / 3,  S = log2 B   [PT-M2]."""
    lg = np.log2(np.asarray(g, dtype=np.float64))
    S = np.log2(np.asarray(B, dtype=np.float64))
    return -0.5 * lg + ((S + 0.5 * lg.sum(axis=-1)) / 3.0)[..., None]


def assign_shapes_fixed(Z, fixed_shape):
    """The fixed-shape block-sparse baseline (R20): every zone takes candidate
    `fixed_shape` (the id order of candidate_shapes), whatever g and rho."""
    edges, vol = candidate_shapes()
    sid = np.full(Z, int(fixed_shape), dtype=np.int64)
    return {"shape_id": sid, "edges": edges[sid], "B": vol[sid].astype(np.int64)}


def assign_shapes(g, rho, tau128=TAU_128, tau256=TAU_256):
    """Nearest candidate (Euclidean distance in log2 space) to l*  [PT-M2], R8, R9.

    Returns dict: shape_id [Z], edges [Z,3], B [Z], ell [Z,3], dist2 [Z,16]
    (inf for candidates of another volume), margin_shape (second best minus
    best squared distance: moving l* by delta shifts the gap between candidates
    c and c' by 2 delta . (e_c - e_c'), so the choice holds while that stays
    below the gap), margin_volume (min |rho - tau|: the distance rho may move
    before B changes).
    """
    edges, vol = candidate_shapes()
    loge = np.log2(edges.astype(np.float64))
    rho = np.asarray(rho, dtype=np.float64)
    B = block_volume(rho, tau128, tau256)
    ell = optimal_log_edges(g, B)
    Z = B.shape[0]
    dist2 = np.full((Z, len(vol)), np.inf)
    sid = np.empty(Z, dtype=np.int64)
    mshape = np.empty(Z)
    for m in range(Z):
        cand = np.nonzero(vol == B[m])[0]
        dd = ((loge[cand] - ell[m]) ** 2).sum(axis=-1)
        dist2[m, cand] = dd
        best = dd.min()
        tied = cand[dd <= best + TIE_TOL]
        sid[m] = tied.min()                     # ids are in lexicographic order inside a volume
        others = np.sort(dd)
        mshape[m] = others[1] - others[0]
    mvol = np.minimum(np.abs(rho - tau128), np.abs(rho - tau256))
    return {"shape_id": sid, "edges": edges[sid], "B": B, "ell": ell, "dist2": dist2,
            "margin_shape": mshape, "margin_volume": mvol}


# --------------------------------------------------------------------------
# Stage 3: permutation into blocks and its inverse                 [NEWS-4], R10
# --------------------------------------------------------------------------
def build_permutation(shape_id, T, H, W):
    """perm[p] = raster index of the token at permuted position p; blk_start [n_blk+1]."""
    edges, _ = candidate_shapes()
    ZT, ZH, ZW = T // ZONE, H // ZONE, W // ZONE
    perm = np.empty(T * H * W, dtype=np.int64)
    starts = [0]
    p = 0
    m = 0
    for zt in range(ZT):
        for zh in range(ZH):
            for zw in range(ZW):
                bT, bH, bW = (int(e) for e in edges[shape_id[m]])
                for bt in range(ZONE // bT):
                    for bh in range(ZONE // bH):
                        for bw in range(ZONE // bW):
                            for ot in range(bT):
                                for oh in range(bH):
                                    for ow in range(bW):
                                        t = zt * ZONE + bt * bT + ot
                                        h = zh * ZONE + bh * bH + oh
                                        w = zw * ZONE + bw * bW + ow
                                        perm[p] = (t * H + h) * W + w
                                        p += 1
                            starts.append(p)
                m += 1
    return perm, np.array(starts, dtype=np.int64)


def permute(X, perm):
    """Raster [N, heads, d] -> blocked [heads, N, d] (row p holds token perm[p])."""
    return np.ascontiguousarray(np.asarray(X)[perm].transpose(1, 0, 2))


def unpermute(Xb, perm):
    """Blocked [heads, N, d] -> raster [N, heads, d] (restore the layout, [NEWS-4])."""
    Xb = np.asarray(Xb)
    out = np.empty((Xb.shape[1], Xb.shape[0], Xb.shape[2]), dtype=Xb.dtype)
    out[perm] = Xb.transpose(1, 0, 2)
    return out


# --------------------------------------------------------------------------
# Stage 4: pooled block scores and probabilities            [PT-M3], R11, R12
# --------------------------------------------------------------------------
def block_pool_score(Qb, Kb, blk_start, scale=None, heads=None):
    """Qbar_i, Kbar_j = block means; P_i = softmax_j(Qbar_i . Kbar_j * scale).

    Qb, Kb: blocked [heads, N, d].  Returns (Qbar, Kbar, P) in fp64 for the
    requested heads (all by default).
    """
    Qb, Kb = np.asarray(Qb), np.asarray(Kb)
    hs = range(Qb.shape[0]) if heads is None else heads
    d = Qb.shape[-1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    nb = len(blk_start) - 1
    Qbar = np.empty((len(hs), nb, d))
    Kbar = np.empty((len(hs), nb, d))
    for a, hh in enumerate(hs):
        q = Qb[hh].astype(np.float64)
        k = Kb[hh].astype(np.float64)
        for i in range(nb):
            Qbar[a, i] = q[blk_start[i]:blk_start[i + 1]].mean(axis=0)
            Kbar[a, i] = k[blk_start[i]:blk_start[i + 1]].mean(axis=0)
    s = np.einsum("hid,hjd->hij", Qbar, Kbar) * scale
    s = s - s.max(axis=-1, keepdims=True)
    e = np.exp(s)
    P = e / e.sum(axis=-1, keepdims=True)
    return Qbar, Kbar, P


# --------------------------------------------------------------------------
# Stage 5: hybrid Top-k / Top-p selection                     [PT-M3], R13, R14
# --------------------------------------------------------------------------
def block_select(P, top_k, top_p):
    """S_i = Top-k(P_i, k) U Top-p(P_i, p), both prefixes of the order (P desc, j asc).

    P: [..., n_blk, n_blk].  Returns dict: sel bool [..., nb, nb], count
    [..., nb], n_k, n_p, and margin [..., nb]: the L1 norm below which no
    perturbation of the row (rounding of P included) can change the selected
    set, and above which one can (inf if none can).
    """
    P = np.asarray(P, dtype=np.float64)
    nb = P.shape[-1]
    order = np.argsort(-P, axis=-1, kind="stable")        # ties keep ascending j
    Ps = np.take_along_axis(P, order, axis=-1)
    csum = np.cumsum(Ps, axis=-1)
    n_k = min(int(top_k), nb)
    if top_p >= 1.0:
        n_p = np.full(P.shape[:-1], nb, dtype=np.int64)
    else:
        reach = csum >= top_p
        n_p = np.where(reach.any(axis=-1), reach.argmax(axis=-1) + 1, nb)
    n = np.maximum(n_k, n_p)
    rank = np.arange(nb)
    sel_sorted = rank < n[..., None]
    sel = np.zeros(P.shape, dtype=bool)
    np.put_along_axis(sel, order, sel_sorted, axis=-1)

    # Decision margin: the L1 size of the smallest perturbation of the row (kept
    # non-negative) that can change S_i.  S_i is the n = max(n_k, n_p) largest
    # values, and the sum of the m largest values moves by at most the L1 norm
    # of a perturbation, so S_i changes only through one of three events:
    #   order: a value outside S_i overtakes one inside (gap between the n-th
    #          and the (n+1)-th value of the order);
    #   up:    the sum of the n largest drops below p, so that n_p exceeds n;
    #   down:  Top-p sets n (n_p > n_k) and the sum of the n-1 largest reaches
    #          p, so that n_p, and with it n, drops by one.
    # When n_p <= n_k a lower n_p leaves n = n_k, so the sum before the Top-p
    # crossing decides nothing there.
    inf = np.full(P.shape[:-1], np.inf)

    def at(a, i):
        return np.take_along_axis(a, np.clip(i, 0, nb - 1)[..., None], -1)[..., 0]

    gap_order = np.where(n < nb, at(Ps, n - 1) - at(Ps, n), inf)
    if top_p < 1.0:
        gap_up = np.where(n < nb, at(csum, n - 1) - top_p, inf)
        gap_down = np.where((n_p > n_k) & (n_p >= 2), top_p - at(csum, n - 2), inf)
    else:
        gap_up = gap_down = inf
    return {"sel": sel, "count": n, "n_k": n_k, "n_p": n_p,
            "margin": np.minimum(gap_order, np.minimum(gap_up, gap_down))}


# --------------------------------------------------------------------------
# Stage 6: exact softmax attention over the selected blocks     [PT-M3], R15
# --------------------------------------------------------------------------
def _keys_of(sel_row, blk_start):
    js = np.nonzero(sel_row)[0]
    if len(js) == 0:
        return np.zeros(0, dtype=np.int64)
    return np.concatenate([np.arange(blk_start[j], blk_start[j + 1]) for j in js])


def _row_block(q, Kh, Vh, idx, scale):
    s = (q @ Kh[idx].T) * scale
    mx = s.max(axis=-1, keepdims=True)
    e = np.exp(s - mx)
    l = e.sum(axis=-1, keepdims=True)
    P = e / l
    return P, P @ Vh[idx], (mx + np.log(l))[:, 0]


def sparse_attention_fwd(Qb, Kb, Vb, blk_start, sel, scale=None, heads=None, q_blocks=None):
    """O and LSE of each query block i over the tokens of the blocks in S_i.

    Qb, Kb, Vb: blocked [heads, N, d]; sel: bool [heads, nb, nb] (rows = query
    blocks).  ``heads`` / ``q_blocks`` restrict the work to a sample; rows not
    computed are NaN.  Returns (O [h_sel, N, d], lse [h_sel, N]) in fp64.
    """
    Qb, Kb, Vb = np.asarray(Qb), np.asarray(Kb), np.asarray(Vb)
    hs = list(range(Qb.shape[0])) if heads is None else list(heads)
    d = Qb.shape[-1]
    N = Qb.shape[1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    nb = len(blk_start) - 1
    qbs = range(nb) if q_blocks is None else q_blocks
    O = np.full((len(hs), N, d), np.nan)
    lse = np.full((len(hs), N), np.nan)
    for a, hh in enumerate(hs):
        Kh = Kb[hh].astype(np.float64)
        Vh = Vb[hh].astype(np.float64)
        for i in qbs:
            r0, r1 = blk_start[i], blk_start[i + 1]
            idx = _keys_of(sel[hh][i], blk_start)
            q = Qb[hh, r0:r1].astype(np.float64)
            if len(idx) == 0:
                O[a, r0:r1] = 0.0
                lse[a, r0:r1] = -np.inf
                continue
            _, o, l = _row_block(q, Kh, Vh, idx, scale)
            O[a, r0:r1] = o
            lse[a, r0:r1] = l
    return O, lse


def sparse_attention_bwd(Qb, Kb, Vb, dOb, blk_start, sel, scale=None, heads=None,
                         q_blocks=None, k_blocks=None):
    """Exact gradients of sparse_attention_fwd under the fixed selection [ZH-FAQ4].

    With P = softmax over the selected keys, O = P V:
      Delta = rowsum(dO * O), dV = P^T dO, dP = dO V^T, dS = P * (dP - Delta),
      dQ = dS K * scale, dK = dS^T Q * scale.  Nothing flows into g, rho or P_i.
    ``q_blocks`` samples the query blocks whose dQ is wanted; ``k_blocks``
    samples the key blocks whose dK/dV are wanted (all query blocks that
    selected them are then visited).  Entries not computed are NaN.
    Returns (dQ, dK, dV) blocked [h_sel, N, d] in fp64.
    """
    Qb, Kb, Vb, dOb = (np.asarray(x) for x in (Qb, Kb, Vb, dOb))
    hs = list(range(Qb.shape[0])) if heads is None else list(heads)
    d = Qb.shape[-1]
    N = Qb.shape[1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    nb = len(blk_start) - 1
    full = q_blocks is None and k_blocks is None
    want_q = set(range(nb)) if full else set(q_blocks or [])
    want_k = list(range(nb)) if full else list(k_blocks or [])
    dQ = np.full((len(hs), N, d), np.nan)
    dK = np.full((len(hs), N, d), np.nan)
    dV = np.full((len(hs), N, d), np.nan)
    for a, hh in enumerate(hs):
        Qh = Qb[hh].astype(np.float64)
        Kh = Kb[hh].astype(np.float64)
        Vh = Vb[hh].astype(np.float64)
        dOh = dOb[hh].astype(np.float64)
        visit = set(want_q)
        if not full:
            selh = np.asarray(sel[hh])
            for j in want_k:
                visit.update(np.nonzero(selh[:, j])[0].tolist())
        gK = np.zeros((N, d))
        gV = np.zeros((N, d))
        for i in sorted(visit):
            r0, r1 = blk_start[i], blk_start[i + 1]
            idx = _keys_of(sel[hh][i], blk_start)
            if len(idx) == 0:
                if i in want_q:
                    dQ[a, r0:r1] = 0.0
                continue
            q = Qh[r0:r1]
            P, o, _ = _row_block(q, Kh, Vh, idx, scale)
            do = dOh[r0:r1]
            delta = (do * o).sum(axis=-1, keepdims=True)
            dP = do @ Vh[idx].T
            dS = P * (dP - delta)
            if i in want_q:
                dQ[a, r0:r1] = (dS @ Kh[idx]) * scale
            np.add.at(gK, idx, (dS.T @ q) * scale)
            np.add.at(gV, idx, P.T @ do)
        for j in want_k:
            r0, r1 = blk_start[j], blk_start[j + 1]
            dK[a, r0:r1] = gK[r0:r1]
            dV[a, r0:r1] = gV[r0:r1]
    return dQ, dK, dV


def sparse_attention_bwd_keys(Qb, Kb, Vb, dOb, blk_start, sel, lse, O, scale=None, heads=None, k_blocks=()):
    """dK, dV of the sampled key blocks from given per-row LSE and O (teacher
    forcing: the forward's LSE and O are taken as known, so that no query row
    has to be re-normalised over its whole key set).  Same gradients as
    sparse_attention_bwd [ZH-FAQ4]:
      P_ij = exp(s_ij - lse_i), Delta_i = dO_i . O_i,
      dV_j = sum_i P_ij dO_i,  dK_j = scale sum_i P_ij (dO_i . V_j - Delta_i) Q_i
    over the query rows i whose block selected the block of key j.
    lse: [h_sel, N], O: [h_sel, N, d] (rows of the heads in ``heads``).
    Returns (dK, dV) blocked [h_sel, N, d] in fp64, NaN outside the sample."""
    Qb, Kb, Vb, dOb = (np.asarray(x) for x in (Qb, Kb, Vb, dOb))
    hs = list(range(Qb.shape[0])) if heads is None else list(heads)
    d = Qb.shape[-1]
    N = Qb.shape[1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    dK = np.full((len(hs), N, d), np.nan)
    dV = np.full((len(hs), N, d), np.nan)
    for a, hh in enumerate(hs):
        selh = np.asarray(sel[hh])
        for j in k_blocks:
            k0, k1 = blk_start[j], blk_start[j + 1]
            Kj = Kb[hh, k0:k1].astype(np.float64)
            Vj = Vb[hh, k0:k1].astype(np.float64)
            gK = np.zeros((k1 - k0, d))
            gV = np.zeros((k1 - k0, d))
            for i in np.nonzero(selh[:, j])[0]:
                r0, r1 = blk_start[i], blk_start[i + 1]
                q = Qb[hh, r0:r1].astype(np.float64)
                do = dOb[hh, r0:r1].astype(np.float64)
                P = np.exp(q @ Kj.T * scale - np.asarray(lse[a, r0:r1], dtype=np.float64)[:, None])
                delta = (do * np.asarray(O[a, r0:r1], dtype=np.float64)).sum(axis=-1, keepdims=True)
                dS = P * (do @ Vj.T - delta)
                gV += P.T @ do
                gK += (dS.T @ q) * scale
            dK[a, k0:k1] = gK
            dV[a, k0:k1] = gV
    return dK, dV


# --------------------------------------------------------------------------
# Whole layer, raster in -> raster out                     [NEWS-4] steps 1-4
# --------------------------------------------------------------------------
def run_layer(Q, K, V, hhat, T, H, W, top_k, top_p, dO=None, eps=EPS,
              tau128=TAU_128, tau256=TAU_256):
    """Every stage in order on small inputs; returns a dict of all intermediates.

    Q, K, V, dO: raster [N, heads, d]; hhat: raster [N, Da].  O, dQ, dK, dV
    come back in raster layout.
    """
    heads, d = Q.shape[1], Q.shape[2]
    ind = zone_indicator(V, hhat, T, H, W, eps)
    shp = assign_shapes(ind["g"], ind["rho"], tau128, tau256)
    perm, blk_start = build_permutation(shp["shape_id"], T, H, W)
    Qb, Kb, Vb = (permute(np.asarray(x, dtype=np.float64), perm) for x in (Q, K, V))
    Qbar, Kbar, P = block_pool_score(Qb, Kb, blk_start)
    sel = block_select(P, top_k, top_p)
    Ob, lse = sparse_attention_fwd(Qb, Kb, Vb, blk_start, sel["sel"])
    out = {"ind": ind, "shapes": shp, "perm": perm, "blk_start": blk_start,
           "Qbar": Qbar, "Kbar": Kbar, "P": P, "select": sel,
           "Ob": Ob, "lse": lse, "O": unpermute(Ob, perm)}
    if dO is not None:
        dOb = permute(np.asarray(dO, dtype=np.float64), perm)
        dQb, dKb, dVb = sparse_attention_bwd(Qb, Kb, Vb, dOb, blk_start, sel["sel"])
        out.update({"dQb": dQb, "dKb": dKb, "dVb": dVb,
                    "dQ": unpermute(dQb, perm), "dK": unpermute(dKb, perm),
                    "dV": unpermute(dVb, perm)})
    return out
