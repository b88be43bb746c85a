"""The dS handoff's index arithmetic (csrc/ds_handoff.cuh), checked on the CPU.

The handoff lets the key-stationary backward kernel store the dS^T blocks it
forms, and the query-stationary kernel read them back through a look-up entry
per unit of its walk.  tests/ds_index_check.cpp compiles the header's functions
for the host and simulates both sides. Every stored value is tagged with its
(head, key granule, key, query granule, query). Every value the look-up side
reads must carry the tag of the dS entry it stands for, or be zero where the
query granule did not select the key granule.

This test then compares the program's entries with an enumeration written here
from the walks' definitions. The walks are the ascending unions of two
granule-level selection rows: a query tile's two rows of the selection, and a
key tile's two rows of its transpose.
"""
import os
import shutil
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "dynamic_block_sparse_macro_b200", "csrc")
SRC = os.path.join(ROOT, "tests", "ds_index_check.cpp")


@pytest.fixture(scope="module")
def checker(tmp_path_factory):
    cxx = shutil.which("g++") or shutil.which("c++")
    if not cxx:
        pytest.skip("no host C++ compiler")
    exe = str(tmp_path_factory.mktemp("ds") / "ds_index_check")
    subprocess.run([cxx, "-O2", "-std=c++17", "-I", CSRC, SRC, "-o", exe], check=True)
    return exe


def selection(rng, heads, MB, density, empty_tiles=(), full_rows=()):
    """Granule-level selection bits [heads][MB][MB] of 1-, 2- and 4-granule blocks."""
    sel = np.zeros((heads, MB, MB), dtype=bool)
    for h in range(heads):
        for q in range(MB):
            g = 0
            while g < MB:
                size = int(rng.choice([1, 2, 4]))
                if rng.random() < density:
                    sel[h, q, g:g + size] = True
                g += size
    for h, t in empty_tiles:
        sel[h, 2 * t:2 * t + 2, :] = False
    for h, q in full_rows:
        sel[h, q, :] = True
    return sel


def pack(sel):
    heads, MB, _ = sel.shape
    SW = (MB + 31) // 32
    words = np.zeros((heads, MB, SW), dtype=np.uint32)
    for w in range(SW):
        chunk = sel[:, :, 32 * w:32 * w + 32]
        bits = (chunk.astype(np.uint64) << np.arange(chunk.shape[2], dtype=np.uint64)).sum(axis=2)
        words[:, :, w] = bits.astype(np.uint32)
    return words, SW


def expected_entries(sel):
    heads, MB, _ = sel.shape
    tph = MB // 2
    # key tiles: ascending query granules that selected either key granule
    uk, base_kv, acc = {}, {}, 0
    for h in range(heads):
        for tk in range(tph):
            qs = [int(q) for q in np.nonzero(sel[h, :, 2 * tk] | sel[h, :, 2 * tk + 1])[0]]
            uk[h, tk] = qs
            base_kv[h, tk] = acc
            acc += len(qs)
    out = []
    for h in range(heads):
        for tq in range(tph):
            ks = np.nonzero(sel[h, 2 * tq] | sel[h, 2 * tq + 1])[0]
            for u, gk in enumerate(int(k) for k in ks):
                ys = []
                for half in range(2):
                    gq = 2 * tq + half
                    if sel[h, gq, gk]:
                        p = 1 + base_kv[h, gk // 2] + uk[h, gk // 2].index(gq)
                        ys.append(128 * p + 64 * (gk & 1))
                    else:
                        ys.append(0)
                out.append((h * tph + tq, u, 64 * gk, ys[0], ys[1]))
    return out, acc


CASES = [
    # heads, MB, density, empty query tiles, full rows
    (1, 8, 0.5, (), ()),
    (2, 40, 0.3, ((0, 3), (1, 0)), ((1, 7),)),
    (1, 72, 0.15, ((0, 35),), ((0, 0), (0, 71))),
    (2, 64, 0.9, (), ()),
    (1, 96, 0.02, ((0, 10), (0, 11)), ()),
    (1, 512, 0.03, ((0, 100),), ((0, 511),)),      # 16 words a row: ranks across many word prefixes
]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_pieces_and_entries_agree(checker, tmp_path, case):
    heads, MB, density, empty, full = CASES[case]
    rng = np.random.default_rng(100 + case)
    sel = selection(rng, heads, MB, density, empty, full)
    words, SW = pack(sel)
    path = tmp_path / "sel.bin"
    with open(path, "wb") as f:
        f.write(np.array([heads, MB, SW], dtype=np.int32).tobytes())
        f.write(words.tobytes())
    r = subprocess.run([checker, str(path)], capture_output=True, text=True, check=True)
    lines = r.stdout.strip().splitlines()
    got = [tuple(int(x) for x in ln.split()[1:]) for ln in lines if ln.startswith("E ")]
    tail = lines[-1].split()
    assert tail[0] == "checked" and tail[2] == "mismatches"
    want, pieces = expected_entries(sel)
    assert got == want
    # every value the look-up reads is the one the key-stationary side stored for it
    assert int(tail[3]) == 0
    assert int(tail[1]) == 2 * 64 * 64 * len(want) > 0
    # pieces and entries stay within the capacities the host carves: the query
    # walk never has more than twice the key walk's units
    assert len(want) <= 2 * pieces
