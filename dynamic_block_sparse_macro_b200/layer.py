"""One Prism video self-attention layer on the GPU, stage by stage through the C ABI.

``PrismSparseAttention`` owns the device buffers of one problem size (torch
allocations: device memory is the only thing torch provides here) and issues
the ABI calls in order on the current CUDA stream:

  forward:  zone_indicator(V, hhat) -> assign_shapes -> permute(Q, K, V)
            -> block_pool_score -> block_select -> sparse_attn_fwd -> unpermute(O)
  backward: permute(dO) -> sparse_attn_bwd -> unpermute(dQ, dK, dV)

Inputs and outputs are raster ``[N, heads, head_dim]`` tensors (``hhat`` is
``[N, audio_dim]``).  No step runs on the CPU and nothing synchronises the
host except where stated.
"""
from __future__ import annotations

import math

import torch

from . import _abi

_TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16}


class PrismSparseAttention:
    def __init__(self, T, H, W, heads, head_dim, audio_dim=64, dtype="bf16", top_k=8, top_p=0.9,
                 eps=1e-6, tau128=0.5, tau256=0.25, scale=None, device="cuda", p_blocks=None,
                 with_backward=True, guidance="joint", fixed_shape=-1):
        self.prob = _abi.problem(T, H, W, heads, head_dim, audio_dim, dtype)
        self.sizes = _abi.query_sizes(self.prob)
        self.dtype = dtype
        self.tdt = _TORCH_DT[dtype]
        self.top_k, self.top_p = int(top_k), float(top_p)
        self.eps, self.tau128, self.tau256 = float(eps), float(tau128), float(tau256)
        # ablations the pages compare against: one guidance term only, one fixed block shape
        self.guidance, self.fixed_shape = guidance, int(fixed_shape)
        self.scale = float(scale) if scale is not None else 1.0 / math.sqrt(head_dim)
        self.heads, self.d = heads, head_dim
        # with_backward=False is the inference path: no backward buffers, no key-major
        # selection, no fp32 copy of O and no LSE
        self.with_backward = bool(with_backward)
        dev = torch.device(device)
        self.device = dev
        s = self.sizes
        N, Z, MB, SW = s.n_tokens, s.n_zones, s.max_blocks, s.sel_words
        f32, i32 = torch.float32, torch.int32
        e = lambda *shape, dt=f32: torch.empty(shape, dtype=dt, device=dev)
        # stage 1-2
        self.g, self.rho, self.abar = e(Z, 3), e(Z), e(Z)
        self.zone_stats = e(Z, 8)
        self.ws_ind = e(max(1, s.ws_indicator), dt=torch.uint8)
        self.shape_id = e(Z, dt=torch.uint8)
        self.perm = e(N, dt=i32)
        self.blk_start = e(MB + 1, dt=i32)
        self.gran_blk = e(MB, dt=i32)
        self.n_blk = e(1, dt=i32)
        self.margin_shape = e(Z, 2)
        # stage 3-5
        self.Qp, self.Kp, self.Vp = (e(heads, N, head_dim, dt=self.tdt) for _ in range(3))
        self.Qbar, self.Kbar = e(heads, MB, head_dim), e(heads, MB, head_dim)
        pb = MB if p_blocks is None else int(p_blocks)
        self.p_blocks = pb
        self.P = e(heads * pb * pb)
        self.sel = e(heads, MB, SW, dt=torch.int32)
        # granule-level selection (the attention kernels' view) and its transpose
        self.gsel = e(heads, MB, SW, dt=torch.int32)
        self.gselT = e(heads, MB, SW, dt=torch.int32) if with_backward else None
        self.sel_count = e(heads, MB, dt=i32)
        self.margin_sel = e(heads, MB)
        self.dev_status = torch.zeros(1, dtype=i32, device=dev)
        # stage 6-7
        self.Op = e(heads, N, head_dim, dt=self.tdt)
        # unrounded O for the backward's Delta (bf16 storage only)
        self.Of32 = e(heads, N, head_dim) if (with_backward and dtype == "bf16") else None
        self.lse = e(heads, N) if with_backward else None
        self.ws_fwd = e(max(16, s.ws_attn_fwd), dt=torch.uint8)
        if with_backward:
            self.dOp = e(heads, N, head_dim, dt=self.tdt)
            self.dQp, self.dKp, self.dVp = (e(heads, N, head_dim, dt=self.tdt) for _ in range(3))
            self.ws_bwd = e(max(16, s.ws_attn_bwd), dt=torch.uint8)

    # ------------------------------------------------------------------ stages
    def plan(self, V, hhat, stream=None):
        """Stages 1-2: zone indicator, shapes, permutation, block table."""
        p = self.prob
        _abi.prism_zone_indicator_ex(p, V, hhat, self.eps, self.guidance, self.g, self.rho, self.abar,
                                     self.zone_stats, self.ws_ind, stream)
        _abi.prism_assign_shapes_ex(p, self.g, self.rho, self.tau128, self.tau256, self.fixed_shape,
                                    self.shape_id, self.perm, None, self.blk_start, self.gran_blk, self.n_blk,
                                    self.margin_shape, stream)

    def select(self, Q, K, V, stream=None):
        """Stages 3-5: permute Q, K, V; pooled probabilities; hybrid selection."""
        p = self.prob
        _abi.prism_permute(p, Q, self.perm, self.Qp, stream)
        _abi.prism_permute(p, K, self.perm, self.Kp, stream)
        _abi.prism_permute(p, V, self.perm, self.Vp, stream)
        _abi.prism_block_pool_score(p, self.Qp, self.Kp, self.blk_start, self.n_blk, self.scale,
                                    self.Qbar, self.Kbar, self.P, stream)
        _abi.prism_block_select(p, self.P, self.blk_start, self.gran_blk, self.n_blk, self.top_k, self.top_p,
                                self.sel, self.sel_count, self.gsel, self.gselT, self.margin_sel,
                                self.dev_status, stream)

    def attend(self, stream=None):
        """Stage 6 on the blocked tensors."""
        _abi.prism_sparse_attn_fwd(self.prob, self.Qp, self.Kp, self.Vp, self.gsel, self.scale, self.Op,
                                   self.lse, self.Of32, self.dev_status, self.ws_fwd, stream)

    def forward(self, Q, K, V, hhat, out=None, stream=None, check=True):
        """Whole forward; returns O in raster layout.

        check: read the device status word once the forward has run (this
        synchronises the stream) and raise if a kernel flagged a condition:
        rows beyond the selection's capacity leave every selection row empty
        and O = 0, and a timed-out wait leaves outputs incomplete.  With
        check=False nothing synchronises; call ``check_status()`` later."""
        self.plan(V, hhat, stream)
        self.select(Q, K, V, stream)
        self.attend(stream)
        if out is None:
            out = torch.empty_like(Q)
        _abi.prism_unpermute(self.prob, self.Op, self.perm, out, stream)
        if check:
            self.check_status(stream)
        return out

    def backward(self, dO, dQ=None, dK=None, dV=None, stream=None, check=True):
        """Stage 7 for the last forward; returns raster (dQ, dK, dV).  ``check``
        as in ``forward``."""
        if not self.with_backward:
            raise RuntimeError("this layer was built for inference (with_backward=False)")
        p = self.prob
        _abi.prism_permute(p, dO, self.perm, self.dOp, stream)
        _abi.prism_sparse_attn_bwd(p, self.Qp, self.Kp, self.Vp, self.Op, self.Of32, self.dOp, self.lse,
                                   self.gsel, self.gselT, self.scale, self.dQp, self.dKp, self.dVp,
                                   self.dev_status, self.ws_bwd, stream)
        outs = []
        for src, dst in ((self.dQp, dQ), (self.dKp, dK), (self.dVp, dV)):
            if dst is None:
                dst = torch.empty_like(dO)
            _abi.prism_unpermute(p, src, self.perm, dst, stream)
            outs.append(dst)
        if check:
            self.check_status(stream)
        return tuple(outs)

    # ------------------------------------------------------------------ memory
    def memory_report(self) -> dict:
        """Device bytes this layer holds, by stage (the caller's raster inputs and
        outputs are not included)."""
        def nb(*ts):
            return int(sum(t.numel() * t.element_size() for t in ts if t is not None))
        rep = {
            "plan": nb(self.g, self.rho, self.abar, self.zone_stats, self.ws_ind, self.shape_id, self.perm,
                       self.blk_start, self.gran_blk, self.n_blk, self.margin_shape),
            "blocked_qkv": nb(self.Qp, self.Kp, self.Vp),
            "scores": nb(self.Qbar, self.Kbar, self.P),
            "selection": nb(self.sel, self.gsel, self.gselT, self.sel_count, self.margin_sel, self.dev_status),
            "forward": nb(self.Op, self.Of32, self.lse, self.ws_fwd),
            "backward": nb(self.dOp, self.dQp, self.dKp, self.dVp, self.ws_bwd) if self.with_backward else 0,
        }
        rep["total"] = sum(rep.values())
        return rep

    # ------------------------------------------------------------------ views
    def num_blocks(self) -> int:
        """Device n_blk (synchronises)."""
        return int(self.n_blk.item())

    def P_view(self):
        nb = self.num_blocks()
        return self.P[: self.heads * nb * nb].view(self.heads, nb, nb)

    def status(self, stream=None) -> int:
        """The device status word (synchronises the stream)."""
        return _abi.prism_read_status(self.dev_status, stream)

    def check_status(self, stream=None) -> None:
        """Raise ``PrismDeviceError`` if a kernel of this layer set a status bit."""
        st = self.status(stream)
        if st:
            raise _abi.PrismDeviceError(st)


class _PrismFn(torch.autograd.Function):
    @staticmethod
    def forward(ctx, Q, K, V, hhat, mod):
        ctx.mod = mod
        return mod.forward(Q.contiguous(), K.contiguous(), V.contiguous(), hhat.contiguous())

    @staticmethod
    def backward(ctx, dO):
        dQ, dK, dV = ctx.mod.backward(dO.contiguous())
        return dQ, dK, dV, None, None


def prism_attention(Q, K, V, hhat, mod: PrismSparseAttention):
    """Autograd entry: O = Prism sparse attention of raster Q, K, V guided by hhat.

    The selection statistics (rho, g, P) are constants for the backward, and
    hhat receives no gradient.
    """
    return _PrismFn.apply(Q, K, V, hhat, mod)
