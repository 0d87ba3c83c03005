"""The debug build of the library (libsta_debug.so: device bounds checks on
every work item, key-block list entry, TMA row coordinate and output row)
on small, odd shapes: ragged text (37 of 256 keys), tiles of 2 or 3 blocks,
several window classes, d = 64 and 128, tile and raster order, backward, and
the SWA and 2-D slide paths.  Every call must report STA_OK (no check fails)
and give the release build's results.
"""
import contextlib

import pytest
import torch

import block_sparse_local_b200 as sta
from block_sparse_local_b200 import workloads

pytestmark = pytest.mark.gpu


@contextlib.contextmanager
def debug_build():
    """Routes the binding's calls to libsta_debug.so for the duration."""
    saved = sta._LIB
    sta._LIB = sta.debug_lib()
    try:
        yield
    finally:
        sta._LIB = saved


def _status_ok():
    # sta.lib() is the build the calls went to (see debug_build)
    code = sta.lib().sta_device_status(None)
    assert code == 0, sta.STATUS.get(code, code)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    assert sta.debug_lib().sta_debug_checks() == 1
    sta.use_pair_kernel(False)


CASES = [
    # T, H, W, tile, windows, text_len, has_text, d, B
    (12, 16, 24, (6, 8, 8), [(1, 2, 3), (2, 2, 2)], 37, True, 64, 2),
    (4, 24, 32, (2, 8, 8), [(1, 3, 3), (2, 2, 4), (9, 9, 9)], 200, True, 128, 1),
    (18, 24, 32, (6, 8, 8), [(1, 3, 3)], 0, False, 64, 1),
]


def _close(a, b):
    err = (a.float() - b.float()).abs()
    return err.max().item() <= 2e-2 and err.mean().item() <= 2e-3


@pytest.mark.parametrize("T,H,W,tile,windows,text_len,has_text,d,B", CASES)
def test_debug_build_forward_backward_lists(T, H, W, tile, windows, text_len, has_text, d, B):
    w = workloads.small_sta_case(T, H, W, tile, windows, text_len, has_text, d=d, B=B, seed=41)
    q, k, v = workloads.sta_inputs(w, device="cuda")
    shape = (T, H, W)
    do = workloads.randn_bf16(q.shape, 4242, device="cuda")
    results = []
    for ctx in (contextlib.nullcontext(), debug_build()):
        with ctx:
            qt, kt, vt, dot = (sta.tile_reorder(x, shape, tile, has_text) for x in (q, k, v, do))
            o, lse = sta.forward(qt, kt, vt, windows, text_len, has_text, shape, tile,
                                 return_lse=True)
            orast = sta.forward_raster(q, k, v, windows, text_len, has_text, shape, tile)
            grads = sta.backward(qt, kt, vt, o, dot, lse, windows, text_len, has_text, shape,
                                 tile)
            counts, ids = sta.build_kv_tile_lists(windows, shape, tile, text_len, has_text)
            back = sta.tile_unreorder(qt, shape, tile, has_text)
            _status_ok()            # the build in use: no bounds check failed
            results.append((qt, o, orast, grads, counts, ids, back))
    rel, dbg = results
    assert torch.equal(rel[0], dbg[0]) and torch.equal(rel[6], dbg[6])     # permutation
    assert torch.equal(rel[4], dbg[4]) and torch.equal(rel[5], dbg[5])     # tile lists
    assert _close(rel[1], dbg[1]) and _close(rel[2], dbg[2])               # forward
    for a, b in zip(rel[3], dbg[3]):                                       # backward
        err = (a.float() - b.float()).abs()
        assert err.max().item() <= 2e-2 * max(1e-6, b.float().abs().max().item())


def test_debug_build_swa_and_slide2d():
    sw = workloads.SwaWorkload("swa_small", 1, 4, 2, 128, 1024, 300, True, 1.0, 7)
    sq, sk, sv = workloads.swa_inputs(sw, device="cuda")
    n, win = 64, 9
    wl = workloads.small_sta_case(1, n, n, (1, n, n), [(1, 1, 1)] * 2, 0, False, d=64, seed=43)
    hq, hk, hv = workloads.sta_inputs(wl, device="cuda")
    outs = []
    for ctx in (contextlib.nullcontext(), debug_build()):
        with ctx:
            a = sta.swa_forward(sq, sk, sv, sw.window, True)
            b = sta.slide_attention_2d(hq, hk, hv, n, win, "hilbert")
            _status_ok()
            outs.append((a, b))
    assert _close(outs[0][0], outs[1][0]) and _close(outs[0][1], outs[1][1])
