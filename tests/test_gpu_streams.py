"""Calls on several streams that share the library's device workspace.

sta_forward and sta_backward keep their tile lists and work plans in a
per-device workspace that every call rewrites.  The library orders a call
after the last call on another stream that used the same workspace (an
event per workspace), so interleaving two problems on two streams must give
exactly the outputs of running them one after another.  The first problem is
the large one, so that its kernels are still running when the second call
rewrites the workspace if the ordering were missing.
"""
import pytest
import torch

import block_sparse_local_b200 as sta
from block_sparse_local_b200 import workloads

pytestmark = pytest.mark.gpu


def _case(w):
    q, k, v = workloads.sta_inputs(w, device="cuda")
    shape = (w.T, w.H, w.W)
    qt, kt, vt = (sta.tile_reorder(x, shape, w.tile, w.has_text) for x in (q, k, v))
    return w, shape, qt, kt, vt


def _fwd(c, out):
    w, shape, qt, kt, vt = c
    return sta.forward(qt, kt, vt, w.windows, w.text_len, w.has_text, shape, w.tile, out=out)


@pytest.fixture(scope="module")
def cases():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    sta.use_pair_kernel(False)
    big = workloads.small_sta_case(30, 48, 80, (6, 8, 8), [(3, 3, 3)] * 4, 200, True,
                                   d=128, seed=31)
    small = workloads.small_sta_case(12, 16, 24, (6, 8, 8), [(1, 2, 3), (2, 2, 2)], 77, True,
                                     d=64, B=2, seed=32)
    return _case(big), _case(small)


def test_forward_on_two_streams_equals_serial(cases):
    big, small = cases
    ref_b = _fwd(big, torch.empty_like(big[2]))
    ref_s = _fwd(small, torch.empty_like(small[2]))
    torch.cuda.synchronize()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    outs = []
    for _ in range(3):
        ob, os_ = torch.empty_like(ref_b), torch.empty_like(ref_s)
        s1.wait_stream(torch.cuda.current_stream())
        s2.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s1):
            _fwd(big, ob)
        with torch.cuda.stream(s2):
            _fwd(small, os_)
        # and the other way round: the big problem after the small one
        ob2, os2 = torch.empty_like(ref_b), torch.empty_like(ref_s)
        with torch.cuda.stream(s2):
            _fwd(small, os2)
        with torch.cuda.stream(s1):
            _fwd(big, ob2)
        outs.append((ob, os_, ob2, os2))
    torch.cuda.synchronize()
    sta.device_status()
    for ob, os_, ob2, os2 in outs:
        assert torch.equal(ob, ref_b) and torch.equal(ob2, ref_b)
        assert torch.equal(os_, ref_s) and torch.equal(os2, ref_s)


def test_backward_on_two_streams_equals_serial(cases):
    big, small = cases
    refs = []
    for c in (big, small):
        w, shape, qt, kt, vt = c
        o, lse = sta.forward(qt, kt, vt, w.windows, w.text_len, w.has_text, shape, w.tile,
                             return_lse=True)
        g = torch.Generator(device="cuda")
        g.manual_seed(77)
        do = torch.randn(qt.shape, generator=g, device="cuda").to(torch.bfloat16)
        grads = sta.backward(qt, kt, vt, o, do, lse, w.windows, w.text_len, w.has_text, shape,
                             w.tile)
        refs.append((o, lse, do, grads))
    torch.cuda.synchronize()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    got = [None, None]
    s1.wait_stream(torch.cuda.current_stream())
    s2.wait_stream(torch.cuda.current_stream())
    for i, (c, st) in enumerate(((big, s1), (small, s2))):
        w, shape, qt, kt, vt = c
        o, lse, do, _ = refs[i]
        with torch.cuda.stream(st):
            got[i] = sta.backward(qt, kt, vt, o, do, lse, w.windows, w.text_len, w.has_text,
                                  shape, w.tile)
    torch.cuda.synchronize()
    sta.device_status()
    for i in range(2):
        for a, b in zip(got[i], refs[i][3]):
            assert torch.equal(a, b)
