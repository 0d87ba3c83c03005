"""sta_forward_noalloc, the entry point for callers that cannot allocate.

Some callers cannot let a library call cudaMalloc: a serving runtime whose
memory pool has reserved the whole device (a stray cudaMalloc can fail or
fragment the pool), or a latency-bound loop that cannot take the implicit
device synchronisation of cudaMalloc / cudaFree.  sta_forward_noalloc keeps
its scratch (KV tile lists and work plan) in a fixed 4 MiB device array
instead.  These tests call it through the C ABI and check that

  * on calls in a row (the same problem twice, then another problem, then
    the first again, so the work plan in the array is kept, replaced and
    replaced back), every output equals sta_forward's bit for bit: both run
    the same kernel on the same plan, so any difference would be scratch
    left over from another call;
  * those calls change the device's free memory by nothing (read with
    cudaMemGetInfo after a first call has loaded the kernels);
  * a problem too large for the array is refused before anything runs.

The file is named so that pytest collects it last.
"""
import ctypes

import pytest
import torch

import block_sparse_local_b200 as sta
from block_sparse_local_b200 import workloads

MAX_ABS, MEAN_ABS = 2e-2, 2e-3
SCRATCH_LIMIT = 5


def _call_noalloc(qt, kt, vt, w, out):
    L = sta.lib()
    wins = (ctypes.c_int * (3 * w.heads))(*[x for win in w.windows for x in win])
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    code = L.sta_forward_noalloc(ctypes.c_void_p(qt.data_ptr()), ctypes.c_void_p(kt.data_ptr()),
                                 ctypes.c_void_p(vt.data_ptr()), ctypes.c_void_p(out.data_ptr()),
                                 w.B, w.heads, w.d, w.T, w.H, w.W,
                                 (ctypes.c_int * 3)(*w.tile), wins, w.text_len, int(w.has_text),
                                 stream)
    assert code == 0, sta.STATUS.get(code, code)


@pytest.mark.gpu
def test_noalloc_matches_forward_on_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    sta.use_pair_kernel(False)   # the kernel sta_forward_noalloc always runs
    base = workloads.VIDEO_TEXT
    first = workloads.small_sta_case(base.T, base.H, base.W, base.tile, [(3, 3, 3)] * 3,
                                     base.text_len, True, d=128, seed=21)
    second = workloads.small_sta_case(12, 16, 24, (6, 8, 8), [(1, 2, 3), (2, 2, 2)], 77, True,
                                      d=64, B=2, seed=22)   # two window classes, text
    cases = {}
    for name, w in (("first", first), ("second", second)):
        q, k, v = workloads.sta_inputs(w, device="cuda")
        shape = (w.T, w.H, w.W)
        qt, kt, vt = (sta.tile_reorder(x, shape, w.tile, w.has_text) for x in (q, k, v))
        ref = sta.forward(qt, kt, vt, w.windows, w.text_len, w.has_text, shape, w.tile)
        cases[name] = (w, qt, kt, vt, ref)
    order = ["first", "first", "second", "first"]
    outs = [torch.empty_like(cases[n][4]) for n in order]
    # a first call loads the kernels (module loading may allocate)
    warm = torch.empty_like(cases["first"][4])
    w, qt, kt, vt, _ = cases["first"]
    _call_noalloc(qt, kt, vt, w, warm)
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    for n, out in zip(order, outs):
        w, qt, kt, vt, _ = cases[n]
        _call_noalloc(qt, kt, vt, w, out)
    torch.cuda.synchronize()
    free_after = torch.cuda.mem_get_info()[0]
    sta.device_status()
    assert free_after == free_before, (free_before, free_after)
    assert torch.equal(warm, cases["first"][4])
    for n, out in zip(order, outs):
        ref = cases[n][4]
        assert torch.equal(out, ref), n
        err = (out.float() - ref.float()).abs()
        assert err.max().item() <= MAX_ABS and err.mean().item() <= MEAN_ABS
        assert torch.isfinite(out.float()).all()


def test_noalloc_refuses_problems_beyond_its_scratch():
    # 16 batch elements x 64 heads of the (36,48,48) grid need about 7 MiB of
    # work plan; refused on the host before any CUDA call.
    L = sta.lib()
    fake = [ctypes.c_void_p((i + 1) << 24) for i in range(4)]
    heads = 64
    wins = (ctypes.c_int * (3 * heads))(*([3, 3, 3] * heads))
    code = L.sta_forward_noalloc(*fake, 16, heads, 128, 36, 48, 48, (ctypes.c_int * 3)(6, 8, 8),
                                 wins, 0, 0, None)
    assert code == SCRATCH_LIMIT
    assert L.sta_status_string(SCRATCH_LIMIT).decode().startswith("STA_ERR_SCRATCH_LIMIT")
