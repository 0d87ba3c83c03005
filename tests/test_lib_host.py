"""CPU checks of the C-ABI library: it loads, exports every symbol that
include/sta.h declares, and rejects bad arguments on the host before touching
the GPU.  Host-side arithmetic (retained pairs) is checked against the oracle.
No kernel is launched here.
"""
import ctypes
import os
import re

import pytest

import block_sparse_local_b200 as sta
from block_sparse_local_b200 import build as sta_build
from block_sparse_local_b200 import workloads
from oracle import sta_oracle, swa_oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    sta_build.build()
    return sta.lib()


def _declared():
    text = open(os.path.join(ROOT, "include", "sta.h")).read()
    return sorted(set(re.findall(r"^\S[^\n(]*?\b(sta_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    names = _declared()
    for want in ("sta_forward", "sta_forward_lse", "sta_tile_reorder", "sta_tile_unreorder",
                 "sta_build_kv_tile_lists", "sta_swa_forward", "sta_device_status",
                 "sta_status_string", "sta_shutdown", "sta_retained_pairs"):
        assert want in names


def test_library_exports_every_declared_symbol(L):
    for name in _declared():
        assert hasattr(L, name), name
    assert set(_declared()) == set(sta.EXPORTED)


def test_debug_build_loads_with_every_symbol_and_its_checks_compiled_in(L):
    # libsta_debug.so is the same library with the device bounds checks
    # (STA_DEBUG=1); sta_debug_checks() tells the two builds apart
    LD = sta.debug_lib()
    for name in _declared():
        assert hasattr(LD, name), name
    assert LD.sta_debug_checks() == 1
    assert L.sta_debug_checks() == 0
    assert LD.sta_status_string(6).decode().startswith("STA_ERR_DEVICE_BOUNDS")


def test_status_strings(L):
    for code, name in sta.STATUS.items():
        assert L.sta_status_string(code).decode().startswith(name)


def _i3(*x):
    return (ctypes.c_int * 3)(*x)


def _wins(*ws):
    flat = [x for w in ws for x in w]
    return (ctypes.c_int * len(flat))(*flat)


FAKE = ctypes.c_void_p(1 << 20)      # never dereferenced: rejected before any launch
FAKE2 = ctypes.c_void_p(2 << 20)
FAKE3 = ctypes.c_void_p(3 << 20)
FAKE4 = ctypes.c_void_p(4 << 20)


@pytest.mark.parametrize("T,H,W,tile,text_len,has_text", [
    (18, 24, 30, (6, 8, 8), 0, 0),     # W not a multiple of the tile
    (18, 24, 32, (0, 8, 8), 0, 0),     # empty tile
    (18, 24, 32, (6, 8, 8), 257, 1),   # text_len > 256
    (18, 24, 32, (6, 8, 8), -1, 1),    # negative text_len
    (18, 24, 32, (6, 8, 8), 0, 2),     # has_text not 0/1
    (0, 24, 32, (6, 8, 8), 0, 0),      # empty grid
])
def test_forward_rejects_bad_geometry(L, T, H, W, tile, text_len, has_text):
    r = L.sta_forward(FAKE, FAKE2, FAKE3, FAKE4, 1, 1, 64, T, H, W, _i3(*tile),
                      _wins((1, 3, 3)), text_len, has_text, None)
    assert r == 1


def test_forward_rejects_bad_windows_and_pointers(L):
    geo = (18, 24, 32, _i3(6, 8, 8))
    assert L.sta_forward(FAKE, FAKE2, FAKE3, FAKE4, 1, 1, 64, *geo, _wins((0, 3, 3)), 0, 0, None) == 1
    assert L.sta_forward(None, FAKE2, FAKE3, FAKE4, 1, 1, 64, *geo, _wins((1, 3, 3)), 0, 0, None) == 1
    assert L.sta_forward(FAKE, FAKE2, FAKE3, FAKE, 1, 1, 64, *geo, _wins((1, 3, 3)), 0, 0, None) == 1
    misaligned = ctypes.c_void_p((1 << 20) + 8)
    assert L.sta_forward(misaligned, FAKE2, FAKE3, FAKE4, 1, 1, 64, *geo, _wins((1, 3, 3)), 0, 0, None) == 1
    assert L.sta_forward(FAKE, FAKE2, FAKE3, FAKE4, 0, 1, 64, *geo, _wins((1, 3, 3)), 0, 0, None) == 1
    assert L.sta_forward_lse(FAKE, FAKE2, FAKE3, FAKE4, None, 1, 1, 64, *geo, _wins((1, 3, 3)), 0, 0, None) == 1


def test_forward_reports_unsupported_shapes(L):
    # d = 96 and a 2x2-token tile (volume 4) are legal STA but not built.
    assert L.sta_forward(FAKE, FAKE2, FAKE3, FAKE4, 1, 1, 96, 18, 24, 32, _i3(6, 8, 8),
                         _wins((1, 3, 3)), 0, 0, None) == 2
    assert L.sta_forward(FAKE, FAKE2, FAKE3, FAKE4, 1, 1, 64, 1, 10, 10, _i3(1, 2, 2),
                         _wins((1, 3, 3)), 0, 0, None) == 2


def test_reorder_and_lists_reject_bad_args(L):
    assert L.sta_tile_reorder(FAKE, FAKE, 1, 1, 64, 18, 24, 32, _i3(6, 8, 8), 0, None) == 1
    assert L.sta_tile_unreorder(FAKE, FAKE2, 1, 1, 64, 18, 24, 31, _i3(6, 8, 8), 0, None) == 1
    assert L.sta_tile_reorder(FAKE, FAKE2, 1, 1, 12, 18, 24, 32, _i3(6, 8, 8), 0, None) == 2
    # max_k too small for the text query row (36 tiles + sentinel)
    assert L.sta_build_kv_tile_lists(FAKE, FAKE2, 20, 1, 18, 24, 32, _i3(6, 8, 8),
                                     _wins((1, 3, 3)), 5, 1, None) == 1
    assert L.sta_build_kv_tile_lists(FAKE, FAKE2, 64, 1, 18, 24, 32, _i3(6, 8, 8),
                                     _wins((1, 3, -1)), 0, 0, None) == 1


def test_host_forward_rejects_bad_args(L):
    geo = (18, 24, 32, _i3(6, 8, 8))
    f = L.sta_forward_raster_host
    assert f(None, FAKE2, FAKE3, FAKE4, 1, 1, 64, *geo, _wins((1, 3, 3)), 0, 0, 0, None) == 1
    assert f(FAKE, FAKE2, FAKE3, FAKE, 1, 1, 64, *geo, _wins((1, 3, 3)), 0, 0, 0, None) == 1
    assert f(FAKE, FAKE2, FAKE3, FAKE4, 1, 0, 64, *geo, _wins((1, 3, 3)), 0, 0, 0, None) == 1
    assert f(FAKE, FAKE2, FAKE3, FAKE4, 1, 1, 64, *geo, _wins((1, 0, 3)), 0, 0, 0, None) == 1
    assert f(FAKE, FAKE2, FAKE3, FAKE4, 1, 1, 64, 18, 24, 30, _i3(6, 8, 8),
             _wins((1, 3, 3)), 0, 0, 0, None) == 1
    assert f(FAKE, FAKE2, FAKE3, FAKE4, 1, 1, 96, *geo, _wins((1, 3, 3)), 0, 0, 0, None) == 2
    # (4, 2, 48) tiles (384 tokens): a 128-row block is not a box of the grid
    assert f(FAKE, FAKE2, FAKE3, FAKE4, 1, 1, 64, 4, 2, 48, _i3(4, 2, 48),
             _wins((1, 1, 1)), 0, 0, 0, None) == 2


def test_swa_rejects_bad_args(L):
    assert L.sta_swa_forward(FAKE, FAKE2, FAKE3, FAKE4, 1, 6, 4, 128, 1024, 64, 1, None) == 1
    assert L.sta_swa_forward(FAKE, FAKE2, FAKE3, FAKE4, 1, 8, 4, 128, 1000, 64, 1, None) == 2
    assert L.sta_swa_forward(FAKE, FAKE2, FAKE3, FAKE4, 1, 8, 4, 128, 1024, 64, 0, None) == 2
    assert L.sta_swa_forward(FAKE, FAKE2, FAKE3, FAKE4, 1, 8, 4, 128, 1024, 0, 1, None) == 1


@pytest.mark.parametrize("w", [workloads.TINY, workloads.VIDEO_TEXT, workloads.VIDEO_ONLY,
                               workloads.IMAGE_2D, workloads.IMAGE_2D_FULL])
def test_retained_pairs_match_oracle(L, w):
    got = sta.retained_pairs(w.B, w.windows, (w.T, w.H, w.W), w.tile, w.text_len, w.has_text)
    want = w.B * sum(sta_oracle.retained_pairs(w.T, w.H, w.W, w.tile, tuple(win), w.text_len,
                                               w.has_text) for win in w.windows)
    assert got == want


def test_swa_pair_count_formula():
    # the bench counts causal-band pairs with the closed form; pin it to the oracle
    S, wdw = 4096, 1000
    assert swa_oracle.swa_retained_pairs(S, wdw) == wdw * (wdw + 1) // 2 + (S - wdw) * wdw
