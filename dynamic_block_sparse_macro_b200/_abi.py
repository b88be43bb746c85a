"""ctypes binding of ``libprism.so`` (the C ABI declared in ``include/prism.h``).

Argument marshalling only: every function takes torch tensors that already
live on the GPU (or raw integer device pointers) and forwards their addresses,
sizes and the current CUDA stream.  Every step of the path runs in the CUDA
library; if it is missing this module raises instead of falling back.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libprism.so")

PRISM_F32, PRISM_BF16 = 0, 1
STATUS = {0: "PRISM_OK", 1: "PRISM_ERR_INVALID_ARG", 2: "PRISM_ERR_SHAPE",
          3: "PRISM_ERR_UNSUPPORTED", 4: "PRISM_ERR_WORKSPACE", 5: "PRISM_ERR_CUDA"}
DEV_TIMEOUT, DEV_BAD_INDEX = 0x1, 0x2

# every symbol include/prism.h declares
EXPORTS = ("prism_query_sizes", "prism_zone_indicator", "prism_assign_shapes", "prism_permute",
           "prism_unpermute", "prism_block_pool_score", "prism_block_select",
           "prism_sparse_attn_fwd", "prism_sparse_attn_bwd", "prism_read_status",
           "prism_status_string", "prism_version", "prism_launch_count",
           "prism_zone_indicator_noalloc", "prism_zone_indicator_ex", "prism_assign_shapes_ex",
           "prism_layer_init", "prism_layer_arena_bytes", "prism_layer_bind", "prism_layer_forward",
           "prism_layer_backward", "prism_layer_step_host", "prism_layer_release", "prism_layer_sizeof",
           "prism_zone_partials", "prism_zone_finalize", "prism_block_pool_score_raster",
           "prism_sparse_attn_fwd_raster", "prism_sparse_attn_bwd_raster", "prism_attn_bwd_ds_bytes",
           "prism_sparse_attn_bwd_ds", "prism_sparse_attn_bwd_raster_ds")
GUIDANCE = {"joint": 0, "video": 1, "audio": 2}
NOALLOC_SCRATCH_BYTES = 2 << 20


class Problem(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("H", ctypes.c_int32), ("W", ctypes.c_int32),
                ("heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("audio_dim", ctypes.c_int32), ("dtype", ctypes.c_int32)]


class Sizes(ctypes.Structure):
    _fields_ = [("n_tokens", ctypes.c_int64), ("n_zones", ctypes.c_int64),
                ("max_blocks", ctypes.c_int64), ("sel_words", ctypes.c_int64),
                ("ws_indicator", ctypes.c_size_t), ("ws_attn_fwd", ctypes.c_size_t),
                ("ws_attn_bwd", ctypes.c_size_t), ("bytes_P_max", ctypes.c_size_t)]


_VP = ctypes.c_void_p


class LayerT(ctypes.Structure):
    """Mirror of prism_layer_t (field order and types as in include/prism.h)."""
    _fields_ = [("prob", Problem), ("top_k", ctypes.c_int32), ("top_p", ctypes.c_float),
                ("eps", ctypes.c_float), ("tau128", ctypes.c_float), ("tau256", ctypes.c_float),
                ("scale", ctypes.c_float), ("guidance", ctypes.c_int32), ("fixed_shape", ctypes.c_int32),
                ("with_backward", ctypes.c_int32), ("with_io", ctypes.c_int32), ("raster", ctypes.c_int32),
                ("p_blocks", ctypes.c_int64),
                ("g", _VP), ("rho", _VP), ("abar", _VP), ("zone_stats", _VP),
                ("ws_ind", _VP), ("ws_ind_bytes", ctypes.c_size_t),
                ("shape_id", _VP), ("perm", _VP), ("blk_start", _VP), ("gran_blk", _VP), ("n_blk", _VP),
                ("margin_shape", _VP), ("Qp", _VP), ("Kp", _VP), ("Vp", _VP),
                ("Qbar", _VP), ("Kbar", _VP), ("P", _VP), ("sel", _VP), ("gsel", _VP), ("gselT", _VP),
                ("sel_count", _VP), ("margin_sel", _VP), ("dev_status", _VP),
                ("Op", _VP), ("Of32", _VP), ("lse", _VP), ("ws_fwd", _VP), ("ws_fwd_bytes", ctypes.c_size_t),
                ("dOp", _VP), ("dQp", _VP), ("dKp", _VP), ("dVp", _VP),
                ("ws_bwd", _VP), ("ws_bwd_bytes", ctypes.c_size_t),
                ("Q", _VP), ("K", _VP), ("V", _VP), ("hhat", _VP), ("O", _VP), ("dO", _VP),
                ("dQ", _VP), ("dK", _VP), ("dV", _VP), ("io_events", _VP)]


class PrismError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} returned {STATUS.get(code, code)}")
        self.code = code


class PrismDeviceError(RuntimeError):
    """A kernel set a bit of the device status word."""

    def __init__(self, bits: int):
        names = [n for b, n in ((DEV_TIMEOUT, "PRISM_DEV_TIMEOUT"), (DEV_BAD_INDEX, "PRISM_DEV_BAD_INDEX"))
                 if bits & b]
        super().__init__(f"device status 0x{bits:x} ({', '.join(names) or 'unknown bit'})")
        self.bits = bits


_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int32
_F = ctypes.c_float
_SZ = ctypes.c_size_t
_PROB = ctypes.POINTER(Problem)

_SIGS = {
    "prism_query_sizes": [_PROB, ctypes.POINTER(Sizes)],
    "prism_zone_indicator": [_PROB, _P, _P, _F, _P, _P, _P, _P, _P, _SZ, _P],
    "prism_zone_indicator_noalloc": [_PROB, _P, _P, _F, _P, _P, _P, _P, _P],
    "prism_assign_shapes": [_PROB, _P, _P, _F, _F, _P, _P, _P, _P, _P, _P, _P, _P],
    "prism_zone_indicator_ex": [_PROB, _P, _P, _F, _I, _P, _P, _P, _P, _P, _SZ, _P],
    "prism_assign_shapes_ex": [_PROB, _P, _P, _F, _F, _I, _P, _P, _P, _P, _P, _P, _P, _P],
    "prism_permute": [_PROB, _P, _P, _P, _P],
    "prism_unpermute": [_PROB, _P, _P, _P, _P],
    "prism_block_pool_score": [_PROB, _P, _P, _P, _P, _F, _P, _P, _P, _P],
    "prism_block_select": [_PROB, _P, _P, _P, _P, _I, _F, _P, _P, _P, _P, _P, _P, _P],
    "prism_sparse_attn_fwd": [_PROB, _P, _P, _P, _P, _F, _P, _P, _P, _P, _P, _SZ, _P],
    "prism_sparse_attn_bwd": [_PROB, _P, _P, _P, _P, _P, _P, _P, _P, _P, _F, _P, _P, _P, _P, _P, _SZ, _P],
    "prism_read_status": [_P, ctypes.POINTER(ctypes.c_uint32), _P],
    "prism_zone_partials": [_PROB, _P, _P, _P, _P, _SZ, _P],
    "prism_block_pool_score_raster": [_PROB, _P, _P, _P, _P, _P, _F, _P, _P, _P, _P],
    "prism_sparse_attn_fwd_raster": [_PROB, _P, _P, _P, _P, _P, _P, _F, _P, _P, _P, _P, _P, _SZ, _P],
    "prism_sparse_attn_bwd_raster": [_PROB, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _F, _P, _P, _P, _P, _P, _SZ,
                                     _P],
    "prism_attn_bwd_ds_bytes": [_PROB, ctypes.c_int64, ctypes.POINTER(ctypes.c_size_t)],
    "prism_sparse_attn_bwd_ds": [_PROB, _P, _P, _P, _P, _P, _P, _P, _P, _P, _F, _P, _P, _P, _P, _P, _SZ, _P, _SZ,
                                 _P],
    "prism_sparse_attn_bwd_raster_ds": [_PROB, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _F, _P, _P, _P, _P, _P, _SZ,
                                        _P, _SZ, _P],
    "prism_zone_finalize": [_PROB, _P, _F, _I, _P, _P, _P, _P, _P, _SZ, _P],
    "prism_layer_init": [ctypes.POINTER(LayerT), _PROB],
    "prism_layer_arena_bytes": [ctypes.POINTER(LayerT), ctypes.POINTER(ctypes.c_size_t)],
    "prism_layer_bind": [ctypes.POINTER(LayerT), _P, _SZ],
    "prism_layer_forward": [ctypes.POINTER(LayerT), _P, _P, _P, _P, _P, _P],
    "prism_layer_backward": [ctypes.POINTER(LayerT), _P, _P, _P, _P, _P, _P, _P, _P],
    "prism_layer_step_host": [ctypes.POINTER(LayerT), _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P],
    "prism_layer_release": [ctypes.POINTER(LayerT)],
}


def lib(path: str | None = None):
    """Load the CUDA library once; raise if it is not built."""
    global _lib
    if _lib is None:
        p = path or os.environ.get("PRISM_LIB", LIB_PATH)
        if not os.path.exists(p):
            raise RuntimeError(f"libprism.so not found at {p}: run `python -m "
                               f"dynamic_block_sparse_macro_b200.build` (no CPU fallback exists)")
        L = ctypes.CDLL(p)
        for name, args in _SIGS.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = ctypes.c_int
        L.prism_status_string.argtypes = [ctypes.c_int]
        L.prism_status_string.restype = ctypes.c_char_p
        L.prism_version.argtypes = []
        L.prism_version.restype = ctypes.c_char_p
        L.prism_launch_count.argtypes = []
        L.prism_launch_count.restype = ctypes.c_ulonglong
        L.prism_layer_sizeof.argtypes = []
        L.prism_layer_sizeof.restype = ctypes.c_size_t
        _lib = L
    return _lib


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn, code):
    if code != 0:
        raise PrismError(fn, code)


def problem(T, H, W, heads, head_dim, audio_dim, dtype) -> Problem:
    dt = {"f32": PRISM_F32, "bf16": PRISM_BF16, PRISM_F32: PRISM_F32, PRISM_BF16: PRISM_BF16}[dtype]
    return Problem(T, H, W, heads, head_dim, audio_dim, dt)


def query_sizes(prob: Problem) -> Sizes:
    s = Sizes()
    _check("prism_query_sizes", lib().prism_query_sizes(ctypes.byref(prob), ctypes.byref(s)))
    return s


def prism_zone_indicator(prob, V, hhat, eps, g, rho, abar, zone_stats, ws, stream=None):
    _check("prism_zone_indicator", lib().prism_zone_indicator(
        ctypes.byref(prob), _ptr(V), _ptr(hhat), eps, _ptr(g), _ptr(rho), _ptr(abar),
        _ptr(zone_stats), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def prism_zone_indicator_ex(prob, V, hhat, eps, guidance, g, rho, abar, zone_stats, ws, stream=None):
    """prism_zone_indicator with one guidance term removed: guidance is
    "joint", "video" or "audio" (or its integer code)."""
    code = GUIDANCE[guidance] if isinstance(guidance, str) else int(guidance)
    _check("prism_zone_indicator_ex", lib().prism_zone_indicator_ex(
        ctypes.byref(prob), _ptr(V), _ptr(hhat), eps, code, _ptr(g), _ptr(rho), _ptr(abar),
        _ptr(zone_stats), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def prism_zone_indicator_noalloc(prob, V, hhat, eps, g, rho, abar, zone_stats, stream=None):
    """Same as prism_zone_indicator with the library's own fixed scratch array,
    for callers that cannot allocate a workspace (see include/prism.h)."""
    _check("prism_zone_indicator_noalloc", lib().prism_zone_indicator_noalloc(
        ctypes.byref(prob), _ptr(V), _ptr(hhat), eps, _ptr(g), _ptr(rho), _ptr(abar),
        _ptr(zone_stats), _stream(stream)))


def prism_assign_shapes(prob, g, rho, tau128, tau256, shape_id, perm, inv_perm, blk_start,
                        gran_blk, n_blk, margin, stream=None):
    _check("prism_assign_shapes", lib().prism_assign_shapes(
        ctypes.byref(prob), _ptr(g), _ptr(rho), tau128, tau256, _ptr(shape_id), _ptr(perm),
        _ptr(inv_perm), _ptr(blk_start), _ptr(gran_blk), _ptr(n_blk), _ptr(margin), _stream(stream)))


def prism_assign_shapes_ex(prob, g, rho, tau128, tau256, fixed_shape, shape_id, perm, inv_perm,
                           blk_start, gran_blk, n_blk, margin, stream=None):
    """prism_assign_shapes with the fixed-shape baseline: fixed_shape = -1 is
    adaptive, 0..15 gives every zone that candidate."""
    _check("prism_assign_shapes_ex", lib().prism_assign_shapes_ex(
        ctypes.byref(prob), _ptr(g), _ptr(rho), tau128, tau256, int(fixed_shape), _ptr(shape_id),
        _ptr(perm), _ptr(inv_perm), _ptr(blk_start), _ptr(gran_blk), _ptr(n_blk), _ptr(margin),
        _stream(stream)))


def prism_permute(prob, src_raster, perm, dst_blocked, stream=None):
    _check("prism_permute", lib().prism_permute(ctypes.byref(prob), _ptr(src_raster), _ptr(perm),
                                                _ptr(dst_blocked), _stream(stream)))


def prism_unpermute(prob, src_blocked, perm, dst_raster, stream=None):
    _check("prism_unpermute", lib().prism_unpermute(ctypes.byref(prob), _ptr(src_blocked), _ptr(perm),
                                                    _ptr(dst_raster), _stream(stream)))


def prism_block_pool_score(prob, Qp, Kp, blk_start, n_blk, scale, Qbar, Kbar, P, stream=None):
    _check("prism_block_pool_score", lib().prism_block_pool_score(
        ctypes.byref(prob), _ptr(Qp), _ptr(Kp), _ptr(blk_start), _ptr(n_blk), scale, _ptr(Qbar),
        _ptr(Kbar), _ptr(P), _stream(stream)))


def prism_block_select(prob, P, blk_start, gran_blk, n_blk, top_k, top_p, sel, sel_count, gsel, gselT,
                       margin, dev_status, stream=None):
    _check("prism_block_select", lib().prism_block_select(
        ctypes.byref(prob), _ptr(P), _ptr(blk_start), _ptr(gran_blk), _ptr(n_blk), int(top_k), float(top_p),
        _ptr(sel), _ptr(sel_count), _ptr(gsel), _ptr(gselT), _ptr(margin), _ptr(dev_status), _stream(stream)))


def prism_sparse_attn_fwd(prob, Qp, Kp, Vp, gsel, scale, Op, lse, o_f32, dev_status, ws=None,
                          stream=None):
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check("prism_sparse_attn_fwd", lib().prism_sparse_attn_fwd(
        ctypes.byref(prob), _ptr(Qp), _ptr(Kp), _ptr(Vp), _ptr(gsel), scale, _ptr(Op), _ptr(lse),
        _ptr(o_f32), _ptr(dev_status), _ptr(ws), nbytes, _stream(stream)))


def prism_sparse_attn_bwd(prob, Qp, Kp, Vp, Op, o_f32, dOp, lse, gsel, gselT, scale, dQp, dKp, dVp,
                          dev_status, ws, stream=None):
    _check("prism_sparse_attn_bwd", lib().prism_sparse_attn_bwd(
        ctypes.byref(prob), _ptr(Qp), _ptr(Kp), _ptr(Vp), _ptr(Op), _ptr(o_f32), _ptr(dOp), _ptr(lse),
        _ptr(gsel), _ptr(gselT), scale, _ptr(dQp), _ptr(dKp), _ptr(dVp), _ptr(dev_status), _ptr(ws),
        ws.numel() * ws.element_size(), _stream(stream)))


def prism_attn_bwd_ds_bytes(prob, pieces: int) -> int:
    out = ctypes.c_size_t(0)
    _check("prism_attn_bwd_ds_bytes", lib().prism_attn_bwd_ds_bytes(ctypes.byref(prob), int(pieces),
                                                                    ctypes.byref(out)))
    return out.value


def prism_sparse_attn_bwd_ds(prob, Qp, Kp, Vp, Op, o_f32, dOp, lse, gsel, gselT, scale, dQp, dKp, dVp,
                             dev_status, ws, ds, stream=None):
    _check("prism_sparse_attn_bwd_ds", lib().prism_sparse_attn_bwd_ds(
        ctypes.byref(prob), _ptr(Qp), _ptr(Kp), _ptr(Vp), _ptr(Op), _ptr(o_f32), _ptr(dOp), _ptr(lse),
        _ptr(gsel), _ptr(gselT), scale, _ptr(dQp), _ptr(dKp), _ptr(dVp), _ptr(dev_status), _ptr(ws),
        ws.numel() * ws.element_size(), _ptr(ds), ds.numel() * ds.element_size(), _stream(stream)))


def prism_read_status(dev_status, stream=None) -> int:
    out = ctypes.c_uint32(0)
    _check("prism_read_status", lib().prism_read_status(_ptr(dev_status), ctypes.byref(out),
                                                        _stream(stream)))
    return out.value


def version() -> str:
    return lib().prism_version().decode()


def launch_count() -> int:
    return int(lib().prism_launch_count())


# ---------------------------------------------------------------- the layer object
def layer_init(prob) -> LayerT:
    L = LayerT()
    _check("prism_layer_init", lib().prism_layer_init(ctypes.byref(L), ctypes.byref(prob)))
    return L


def layer_arena_bytes(L: LayerT) -> int:
    n = ctypes.c_size_t(0)
    _check("prism_layer_arena_bytes", lib().prism_layer_arena_bytes(ctypes.byref(L), ctypes.byref(n)))
    return n.value


def prism_layer_forward(L: LayerT, Q, K, V, hhat, O, stream=None):
    _check("prism_layer_forward", lib().prism_layer_forward(ctypes.byref(L), _ptr(Q), _ptr(K), _ptr(V),
                                                            _ptr(hhat), _ptr(O), _stream(stream)))


def prism_layer_backward(L: LayerT, Q, K, V, dO, dQ, dK, dV, stream=None):
    _check("prism_layer_backward", lib().prism_layer_backward(ctypes.byref(L), _ptr(Q), _ptr(K), _ptr(V), _ptr(dO),
                                                              _ptr(dQ), _ptr(dK), _ptr(dV), _stream(stream)))


def prism_layer_step_host(L: LayerT, hQ, hK, hV, hhhat, hdO, hO, hdQ, hdK, hdV, compute, h2d, d2h):
    """One step from host (pinned CPU tensor) buffers; see include/prism.h."""
    _check("prism_layer_step_host", lib().prism_layer_step_host(
        ctypes.byref(L), _ptr(hQ), _ptr(hK), _ptr(hV), _ptr(hhhat), _ptr(hdO), _ptr(hO), _ptr(hdQ), _ptr(hdK),
        _ptr(hdV), _stream(compute), _stream(h2d), _stream(d2h)))


def prism_layer_release(L: LayerT):
    """Destroy the CUDA events a host-buffer step created in L (see include/prism.h)."""
    _check("prism_layer_release", lib().prism_layer_release(ctypes.byref(L)))


# ---------------------------------------------------------------- head-sharded indicator
def prism_zone_partials(prob_local, V_local, hhat, partials, ws, stream=None):
    _check("prism_zone_partials", lib().prism_zone_partials(ctypes.byref(prob_local), _ptr(V_local), _ptr(hhat),
                                                            _ptr(partials), _ptr(ws), ws.numel(),
                                                            _stream(stream)))


def prism_zone_finalize(prob, partials, eps, guidance, g, rho, abar, zone_stats, ws, stream=None):
    _check("prism_zone_finalize", lib().prism_zone_finalize(
        ctypes.byref(prob), _ptr(partials), eps, GUIDANCE.get(guidance, guidance), _ptr(g), _ptr(rho), _ptr(abar),
        _ptr(zone_stats), _ptr(ws), ws.numel(), _stream(stream)))


# ---------------------------------------------------------------- raster (no blocked copies)
def prism_block_pool_score_raster(prob, Q, K, perm, blk_start, n_blk, scale, Qbar, Kbar, P, stream=None):
    _check("prism_block_pool_score_raster", lib().prism_block_pool_score_raster(
        ctypes.byref(prob), _ptr(Q), _ptr(K), _ptr(perm), _ptr(blk_start), _ptr(n_blk), scale, _ptr(Qbar),
        _ptr(Kbar), _ptr(P), _stream(stream)))


def prism_sparse_attn_fwd_raster(prob, Q, K, V, perm, shape_id, gsel, scale, O, lse, o_f32, dev_status, ws,
                                 stream=None):
    _check("prism_sparse_attn_fwd_raster", lib().prism_sparse_attn_fwd_raster(
        ctypes.byref(prob), _ptr(Q), _ptr(K), _ptr(V), _ptr(perm), _ptr(shape_id), _ptr(gsel), scale, _ptr(O),
        _ptr(lse), _ptr(o_f32), _ptr(dev_status), _ptr(ws), ws.numel() if ws is not None else 0, _stream(stream)))


def prism_sparse_attn_bwd_raster(prob, Q, K, V, o_f32, dO, lse, perm, shape_id, gsel, gselT, scale, dQ, dK, dV,
                                 dev_status, ws, stream=None):
    _check("prism_sparse_attn_bwd_raster", lib().prism_sparse_attn_bwd_raster(
        ctypes.byref(prob), _ptr(Q), _ptr(K), _ptr(V), _ptr(o_f32), _ptr(dO), _ptr(lse), _ptr(perm), _ptr(shape_id),
        _ptr(gsel), _ptr(gselT), scale, _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(dev_status), _ptr(ws), ws.numel(),
        _stream(stream)))


def prism_sparse_attn_bwd_raster_ds(prob, Q, K, V, o_f32, dO, lse, perm, shape_id, gsel, gselT, scale, dQ, dK,
                                    dV, dev_status, ws, ds, stream=None):
    _check("prism_sparse_attn_bwd_raster_ds", lib().prism_sparse_attn_bwd_raster_ds(
        ctypes.byref(prob), _ptr(Q), _ptr(K), _ptr(V), _ptr(o_f32), _ptr(dO), _ptr(lse), _ptr(perm), _ptr(shape_id),
        _ptr(gsel), _ptr(gselT), scale, _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(dev_status), _ptr(ws),
        ws.numel() * ws.element_size(), _ptr(ds), ds.numel() * ds.element_size(), _stream(stream)))
