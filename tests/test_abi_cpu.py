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
