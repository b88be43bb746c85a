"""One Prism video self-attention layer on the GPU, stage by stage through the C ABI.

``PrismSparseAttention`` owns the device buffers of one problem size (torch
allocations: device memory is the only thing torch provides here), describes
them to the library as one ``prism_layer_t`` and runs the stages on the current
CUDA stream through the library's layer calls:

  forward:  zone_indicator(V, hhat) -> assign_shapes -> permute(Q, K, V)
            -> block_pool_score -> block_select -> sparse_attn_fwd -> unpermute(O)
  backward: permute(dO) -> sparse_attn_bwd -> unpermute(dQ, dK, dV)

The per-stage methods (``plan``, ``select``, ``attend``) issue the same stage
calls one by one, for callers that time or inspect a stage.

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
                 with_backward=True, guidance="joint", fixed_shape=-1, raster=False):
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
        # raster=True: the attention reads Q, K, V, dO and writes O, dQ, dK, dV in place
        # through the permutation (no blocked copies); bf16 only
        self.raster = bool(raster)
        if self.raster and dtype != "bf16":
            raise ValueError("raster=True needs dtype='bf16'")
        self._fwd_inputs = None
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
        if self.raster:
            self.Qp = self.Kp = self.Vp = None
        else:
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
        self.Op = None if self.raster else e(heads, N, head_dim, dt=self.tdt)
        # unrounded O for the backward's Delta (bf16 storage only)
        self.Of32 = e(heads, N, head_dim) if (with_backward and dtype == "bf16") else None
        self.lse = e(heads, N) if with_backward else None
        self.ws_fwd = e(max(16, s.ws_attn_fwd), dt=torch.uint8)
        if with_backward:
            if self.raster:
                self.dOp = self.dQp = self.dKp = self.dVp = None
            else:
                self.dOp = e(heads, N, head_dim, dt=self.tdt)
                self.dQp, self.dKp, self.dVp = (e(heads, N, head_dim, dt=self.tdt) for _ in range(3))
            self.ws_bwd = e(max(16, s.ws_attn_bwd), dt=torch.uint8)
        self.L = self._describe()

    def _describe(self):
        """The library's view of this layer: parameters and buffer addresses."""
        L = _abi.layer_init(self.prob)
        L.top_k, L.top_p, L.eps = self.top_k, self.top_p, self.eps
        L.tau128, L.tau256, L.scale = self.tau128, self.tau256, self.scale
        L.guidance, L.fixed_shape = _abi.GUIDANCE[self.guidance], self.fixed_shape
        L.with_backward, L.with_io, L.p_blocks = int(self.with_backward), 0, self.p_blocks
        L.raster = int(self.raster)
        for name in ("g", "rho", "abar", "zone_stats", "ws_ind", "shape_id", "perm", "blk_start", "gran_blk",
                     "n_blk", "margin_shape", "Qp", "Kp", "Vp", "Qbar", "Kbar", "P", "sel", "gsel", "gselT",
                     "sel_count", "margin_sel", "dev_status", "Op", "Of32", "lse", "ws_fwd"):
            t = getattr(self, name)
            setattr(L, name, t.data_ptr() if t is not None else None)
        L.ws_ind_bytes = self.ws_ind.numel()
        L.ws_fwd_bytes = self.ws_fwd.numel()
        if self.with_backward:
            for name in ("dOp", "dQp", "dKp", "dVp", "ws_bwd"):
                t = getattr(self, name)
                setattr(L, name, t.data_ptr() if t is not None else None)
            L.ws_bwd_bytes = self.ws_bwd.numel()
        return L

    def attach_io(self, Q, K, V, hhat, O, dO=None, dQ=None, dK=None, dV=None):
        """Device raster tensors that ``step_host`` uploads into and downloads from."""
        self._io = (Q, K, V, hhat, O, dO, dQ, dK, dV)
        for name, t in zip(("Q", "K", "V", "hhat", "O", "dO", "dQ", "dK", "dV"), self._io):
            setattr(self.L, name, t.data_ptr() if t is not None else None)
        self.L.with_io = 1

    def step_host(self, hQ, hK, hV, hhhat, hdO, hO, hdQ, hdK, hdV, compute, h2d, d2h):
        """One whole step from pinned host tensors through the library's host-buffer
        call (uploads, forward, backward, downloads on three streams).  Asynchronous:
        the host outputs are final once ``d2h`` has passed this call."""
        _abi.prism_layer_step_host(self.L, hQ, hK, hV, hhhat, hdO, hO, hdQ, hdK, hdV, compute, h2d, d2h)

    def release(self):
        """Destroy the CUDA events the host-buffer step created (once its last call has completed)."""
        if getattr(self, "L", None) is not None and self.L.io_events:
            _abi.prism_layer_release(self.L)

    def __del__(self):
        try:
            self.release()
        except Exception:       # interpreter shutdown: the library may be gone already
            pass

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

    def select_raster(self, Q, K, stream=None):
        """Stages 4-5 reading raster Q, K through the permutation (no blocked copies)."""
        p = self.prob
        _abi.prism_block_pool_score_raster(p, Q, K, self.perm, self.blk_start, self.n_blk, self.scale, self.Qbar,
                                           self.Kbar, self.P, stream)
        _abi.prism_block_select(p, self.P, self.blk_start, self.gran_blk, self.n_blk, self.top_k, self.top_p,
                                self.sel, self.sel_count, self.gsel, self.gselT, self.margin_sel, self.dev_status,
                                stream)

    def attend_raster(self, Q, K, V, out, stream=None):
        """Stage 6 from raster Q, K, V into raster O (``out``)."""
        _abi.prism_sparse_attn_fwd_raster(self.prob, Q, K, V, self.perm, self.shape_id, self.gsel, self.scale, out,
                                          self.lse, self.Of32, self.dev_status, self.ws_fwd, stream)

    def attend_backward_raster(self, Q, K, V, dO, dQ, dK, dV, stream=None):
        """Stage 7 from raster Q, K, V, dO into raster dQ, dK, dV."""
        _abi.prism_sparse_attn_bwd_raster(self.prob, Q, K, V, self.Of32, dO, self.lse, self.perm, self.shape_id,
                                          self.gsel, self.gselT, self.scale, dQ, dK, dV, self.dev_status, self.ws_bwd,
                                          stream)

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
        if out is None:
            out = torch.empty_like(Q)
        _abi.prism_layer_forward(self.L, Q, K, V, hhat, out, stream)
        if self.raster and self.with_backward:
            self._fwd_inputs = (Q, K, V)          # the raster backward reads them again
        if check:
            self.check_status(stream)
        return out

    def backward(self, dO, dQ=None, dK=None, dV=None, stream=None, check=True):
        """Stage 7 for the last forward; returns raster (dQ, dK, dV).  ``check``
        as in ``forward``."""
        if not self.with_backward:
            raise RuntimeError("this layer was built for inference (with_backward=False)")
        outs = [t if t is not None else torch.empty_like(dO) for t in (dQ, dK, dV)]
        q, k, v = self._fwd_inputs if self.raster else (None, None, None)
        if self.raster and q is None:
            raise RuntimeError("backward before forward")
        _abi.prism_layer_backward(self.L, q, k, v, dO, *outs, stream)
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
