"""The C-ABI library loads, exports every symbol include/prism.h declares, and
rejects bad arguments before any launch (no GPU needed: nothing here computes)."""
import ctypes
import os
import re
import subprocess

import pytest

from dynamic_block_sparse_macro_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "prism.h")


@pytest.fixture(scope="module")
def L():
    from dynamic_block_sparse_macro_b200 import build
    build.build()
    return _abi.lib()


def _declared():
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(prism_[a-z0-9_]+)\s*\(", txt)))


def test_header_declares_exactly_the_binding_exports():
    assert _declared() == sorted(_abi.EXPORTS)


def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", _abi.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (prism_[a-z0-9_]+)", out))
    for name in _declared():
        assert name in exported, name
        assert hasattr(L, name)


def test_version_and_status_strings(L):
    assert "sm_100a" in _abi.version()
    for code in range(6):
        assert L.prism_status_string(code)


def test_query_sizes_2k():
    s = _abi.query_sizes(_abi.problem(32, 72, 128, 24, 128, 64, "bf16"))
    assert (s.n_tokens, s.n_zones, s.max_blocks, s.sel_words) == (294912, 576, 4608, 144)
    assert s.bytes_P_max == 24 * 4608 * 4608 * 4
    assert s.ws_attn_bwd >= 24 * 294912 * 4


@pytest.mark.parametrize("T,H,W,heads,d,Da,dt,code", [
    (30, 72, 128, 24, 128, 64, "bf16", 2),      # axis not a multiple of 8
    (0, 8, 8, 1, 64, 64, "f32", 2),
    (8, 8, 8, 1, 96, 64, "f32", 3),             # head_dim
    (8, 8, 8, 65, 64, 64, "f32", 3),            # heads
    (8, 8, 8, 1, 64, 0, "f32", 3),              # audio_dim
    (256, 256, 512, 1, 64, 64, "f32", 3),       # N > 2^24
])
def test_bad_problems_rejected(L, T, H, W, heads, d, Da, dt, code):
    p = _abi.problem(T, H, W, heads, d, Da, dt)
    s = _abi.Sizes()
    assert L.prism_query_sizes(ctypes.byref(p), ctypes.byref(s)) == code


def test_bad_pointers_rejected_before_launch(L):
    p = _abi.problem(8, 8, 8, 1, 64, 64, "f32")
    fake = 1 << 40                                 # aligned, never dereferenced on the host
    # null output
    assert L.prism_permute(ctypes.byref(p), fake, fake, None, None) == 1
    # misaligned pointer
    assert L.prism_permute(ctypes.byref(p), fake + 4, fake, fake + 64, None) == 1
    # in place is refused
    assert L.prism_permute(ctypes.byref(p), fake, fake, fake, None) == 1
    # bad scalars
    assert L.prism_block_select(ctypes.byref(p), fake, fake, fake, fake, -1, 0.9, fake, fake, fake, None, None,
                                fake, None) == 1
    assert L.prism_block_select(ctypes.byref(p), fake, fake, fake, fake, 0, 0.0, fake, fake, fake, None, None,
                                fake, None) == 1
    # ablation options out of range
    assert L.prism_zone_indicator_ex(ctypes.byref(p), fake, fake, 1e-6, 3, fake, fake, fake, None, fake, 1 << 30,
                                     None) == 1
    assert L.prism_assign_shapes_ex(ctypes.byref(p), fake, fake, 0.5, 0.25, 16, fake, fake, None, fake, fake,
                                    fake, None, None) == 1
    assert L.prism_assign_shapes_ex(ctypes.byref(p), fake, fake, 0.5, 0.25, -2, fake, fake, None, fake, fake,
                                    fake, None, None) == 1
    assert L.prism_block_select(ctypes.byref(p), fake, fake, fake, fake, 4, float("nan"), fake, fake, fake, None,
                                None, fake, None) == 1
    # granule-level selection is required
    assert L.prism_block_select(ctypes.byref(p), fake, fake, fake, fake, 4, 0.9, fake, fake, None, None, None,
                                fake, None) == 1
    assert L.prism_zone_indicator(ctypes.byref(p), fake, fake, 0.0, fake, fake, fake, None, fake, 1 << 20, None) == 1
    # workspace too small
    assert L.prism_zone_indicator(ctypes.byref(p), fake, fake, 1e-6, fake, fake, fake, None, fake, 4, None) == 4
    assert L.prism_assign_shapes(ctypes.byref(p), fake, fake, 0.25, 0.5, fake, fake, None, fake, fake, fake,
                                 None, None) == 1      # tau256 > tau128


def test_ds_handoff_sizes_and_checks(L):
    """The dS handoff buffer: a fixed part (gate, the plans' unit prefixes, the key
    tiles' word prefixes, alignment) plus, per piece, 16 KB of dS^T and two 16-byte
    look-up entries; bad buffers are refused before any launch."""
    p = _abi.problem(32, 72, 128, 24, 128, 64, "bf16")
    s = _abi.query_sizes(p)
    tiles = 24 * s.n_tokens // 128
    a16 = lambda b: (b + 15) // 16 * 16
    fixed = 256 + 2 * a16(8 * tiles) + a16(4 * tiles * s.sel_words) + 256
    for pieces in (1, 1000, 2_215_883):
        assert _abi.prism_attn_bwd_ds_bytes(p, pieces) == fixed + 16384 + pieces * (16384 + 32)
    out = ctypes.c_size_t(0)
    for bad in (0, -1, 1 << 24):
        assert L.prism_attn_bwd_ds_bytes(ctypes.byref(p), bad, ctypes.byref(out)) == 1
    fake, ws = 1 << 40, s.ws_attn_bwd
    args = [fake] * 9 + [1.0 / 128 ** 0.5] + [fake] * 5
    need = _abi.prism_attn_bwd_ds_bytes(p, 1)
    bwd = L.prism_sparse_attn_bwd_ds
    assert bwd(ctypes.byref(p), *args, ws, None, need, None) == 1            # no buffer
    assert bwd(ctypes.byref(p), *args, ws, fake + 8, need, None) == 1        # misaligned
    assert bwd(ctypes.byref(p), *args, ws, fake, need - 1, None) == 4        # too small for one piece
    assert bwd(ctypes.byref(p), *args, ws - 1, fake, need, None) == 4        # workspace too small
    pf = _abi.problem(32, 72, 128, 24, 128, 64, "f32")
    assert bwd(ctypes.byref(pf), *args, _abi.query_sizes(pf).ws_attn_bwd, fake, need, None) == 3
    rargs = [fake] * 10 + [1.0 / 128 ** 0.5] + [fake] * 5
    assert L.prism_sparse_attn_bwd_raster_ds(ctypes.byref(p), *rargs, ws, fake, need - 1, None) == 4
    assert L.prism_sparse_attn_bwd_raster_ds(ctypes.byref(p), *rargs, ws, None, need, None) == 1


# ---------------------------------------------------------------- the layer object
def test_layer_struct_matches_the_c_compiler(L):
    # the C driver prints sizeof and every field offset as the C compiler lays them out
    from dynamic_block_sparse_macro_b200 import build
    drv = build.build_driver()
    out = subprocess.run([drv, "offsets"], capture_output=True, text=True, check=True).stdout.split("\n")
    got = dict(line.split() for line in out if line.strip())
    assert int(got.pop("sizeof")) == ctypes.sizeof(_abi.LayerT) == L.prism_layer_sizeof()
    names = [f[0] for f in _abi.LayerT._fields_]
    assert sorted(got) == sorted(names)
    for name in names:
        assert int(got[name]) == getattr(_abi.LayerT, name).offset, name


def test_layer_init_defaults_and_arena_carving(L):
    p = _abi.problem(32, 72, 128, 24, 128, 64, "bf16")
    lay = _abi.layer_init(p)
    assert (lay.top_k, round(lay.top_p, 6), lay.fixed_shape, lay.with_backward, lay.with_io) == (8, 0.9, -1, 1, 0)
    assert abs(lay.scale - 128 ** -0.5) < 1e-7
    sz = _abi.query_sizes(p)
    train = _abi.layer_arena_bytes(lay)
    lay.with_backward = 0
    infer = _abi.layer_arena_bytes(lay)
    lay.with_backward, lay.with_io = 1, 1
    io = _abi.layer_arena_bytes(lay)
    tok = 294912 * 24 * 128 * 2
    assert infer < train < io
    # the training layer holds at least Qp, Kp, Vp, Op, dOp, dQp, dKp, dVp, fp32 O, P, workspaces
    assert train >= 8 * tok + 2 * tok + sz.bytes_P_max + sz.ws_attn_bwd + sz.ws_attn_fwd
    assert io - train >= 8 * tok                     # Q K V O dO dQ dK dV (+ hhat)
    # bind on a fake, aligned device address: host-only pointer arithmetic
    base = 1 << 40
    assert L.prism_layer_bind(ctypes.byref(lay), base, io - 1) == 4              # too small
    assert L.prism_layer_bind(ctypes.byref(lay), base + 16, io) == 1             # misaligned
    assert L.prism_layer_bind(ctypes.byref(lay), base, io) == 0
    ptrs = [getattr(lay, f[0]) for f in _abi.LayerT._fields_ if f[1] is ctypes.c_void_p and f[0] != "io_events"]
    assert all(q is not None and base <= q < base + io and q % 256 == 0 for q in ptrs)
    assert lay.io_events is None                      # the host-buffer step's events: none until one runs
    assert L.prism_layer_release(ctypes.byref(lay)) == 0     # nothing to release: a no-op
    assert len(set(ptrs)) == len(ptrs)
    assert lay.ws_bwd_bytes == sz.ws_attn_bwd and lay.ws_fwd_bytes == sz.ws_attn_fwd
    # bad parameters are refused before anything is carved
    lay.top_p = 0.0
    assert L.prism_layer_arena_bytes(ctypes.byref(lay), ctypes.byref(ctypes.c_size_t())) == 1
