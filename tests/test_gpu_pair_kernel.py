"""GPU parity of the CTA-pair kernel of the d = 128 STA forward (a cluster of
two CTAs per pair of SMs, tcgen05 MMAs with M = 256 issued for both SMs,
three score buffers), selected with the library's kernel hook.

Same checks as for the one-SM kernel: against the float64 oracle on small
grids (tile and raster order, partial text, several window classes, two
batch elements, log-sum-exp), and at the full video+text size on the rows the
oracle can compute one by one, plus agreement with the one-SM kernel on the
whole output.  Tolerance: max-abs <= 2e-2, mean-abs <= 2e-3 per (b, h).
"""
import numpy as np
import pytest
import torch

import block_sparse_local_b200 as sta
from block_sparse_local_b200 import workloads
from oracle import perm_oracle, sta_oracle

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 2e-2, 2e-3


@pytest.fixture(autouse=True)
def _pair_kernel():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    sta.use_pair_kernel(True)
    yield
    sta.use_pair_kernel(False)


def _oracle(w, q, k, v, rows=None):
    q64, k64, v64 = (x.double().numpy() for x in (q, k, v))
    return sta_oracle.sta_forward_batched(q64, k64, v64, w.T, w.H, w.W, w.tile, w.windows,
                                          w.text_len, w.has_text, rows=rows)


def _compare(got, res):
    for (b, h), (ref, _) in res.items():
        err = np.abs(got[b, h] - ref)
        assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (b, h, err.max(), err.mean())


CASES = [
    # (T,H,W), tile, windows, text_len, has_text, B
    ((12, 16, 24), (6, 8, 8), [(2, 2, 2), (1, 1, 3)], 200, True, 1),
    ((12, 16, 24), (6, 8, 8), [(1, 2, 3)], 1, True, 2),
    ((12, 16, 24), (6, 8, 8), [(3, 3, 3)], 256, True, 1),
    ((12, 16, 24), (6, 8, 8), [(1, 1, 1)], 0, True, 1),
    ((4, 24, 32), (2, 8, 8), [(1, 3, 3), (2, 2, 4)], 37, True, 1),
    ((1, 64, 64), (1, 16, 16), [(1, 3, 3)], 0, False, 2),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0]}-{c[1]}-t{c[3]}-B{c[5]}")
@pytest.mark.parametrize("order", ["tile", "raster"])
def test_pair_kernel_matches_oracle(case, order):
    shape, tile, windows, text_len, has_text, B = case
    w = workloads.small_sta_case(*shape, tile, windows, text_len, has_text, d=128, B=B,
                                 seed=23)
    q, k, v = workloads.sta_inputs(w)
    if order == "raster":
        out, lse = sta.forward_raster(q.cuda(), k.cuda(), v.cuda(), w.windows, w.text_len,
                                      w.has_text, shape, w.tile, return_lse=True)
        sta.device_status()
        got, got_lse = out.float().cpu().numpy(), lse.cpu().numpy()
    else:
        qt, kt, vt = (torch.from_numpy(perm_oracle.reorder(x.view(torch.int16).numpy(), *shape,
                                                           w.tile, w.has_text))
                      .view(torch.bfloat16) for x in (q, k, v))
        ot, lt = sta.forward(qt.cuda(), kt.cuda(), vt.cuda(), w.windows, w.text_len,
                             w.has_text, shape, w.tile, return_lse=True)
        sta.device_status()
        got = perm_oracle.unreorder(ot.float().cpu().numpy(), *shape, w.tile, w.has_text)
        got_lse = perm_oracle.unreorder(lt.cpu().numpy()[..., None], *shape, w.tile,
                                        w.has_text)[..., 0]
    res = _oracle(w, q, k, v)
    _compare(got, res)
    for (b, h), (_, ref_lse) in res.items():
        assert np.abs(got_lse[b, h] - ref_lse).max() < 1e-2


def test_pair_kernel_full_video_text_workload():
    # the benchmarked workload: sampled rows against the oracle, every row
    # against the one-SM kernel
    w = workloads.VIDEO_TEXT
    shape = (w.T, w.H, w.W)
    q, k, v = workloads.sta_inputs(w, device="cuda")
    out = sta.forward_raster(q, k, v, w.windows, w.text_len, w.has_text, shape, w.tile)
    sta.device_status()
    sta.use_pair_kernel(False)
    ref = sta.forward_raster(q, k, v, w.windows, w.text_len, w.has_text, shape, w.tile)
    sta.device_status()
    diff = (out.float() - ref.float()).abs()
    assert diff.max().item() <= MAX_ABS and diff.mean().item() <= 1e-4
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([rng.integers(0, w.L_v, size=384),
                                     np.arange(w.L_v, w.S)]))
    for h in (0, 17):
        q64, k64, v64 = (x[0, h].double().cpu().numpy() for x in (q, k, v))
        want, _ = sta_oracle.sta_forward_rows(q64, k64, v64, w.T, w.H, w.W, w.tile,
                                              tuple(w.windows[h]), w.text_len, w.has_text,
                                              rows=rows)
        err = np.abs(out[0, h].float().cpu().numpy()[rows] - want)
        assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (h, err.max(), err.mean())


def test_pair_kernel_many_items_per_cluster():
    # 2 x 8 slices of a 2 x 2 x 3 tile grid: ~300 work items, several per
    # persistent cluster, so the pipeline runs across item boundaries
    wins = [(1, 1, 1), (2, 2, 3), (1, 2, 2), (2, 1, 3)] * 2
    w = workloads.small_sta_case(12, 16, 24, (6, 8, 8), wins, 77, True, d=128, B=2, seed=29)
    shape = (w.T, w.H, w.W)
    q, k, v = workloads.sta_inputs(w)
    out = sta.forward_raster(q.cuda(), k.cuda(), v.cuda(), w.windows, w.text_len, w.has_text,
                             shape, w.tile)
    sta.device_status()
    _compare(out.float().cpu().numpy(), _oracle(w, q, k, v))
    sta.use_pair_kernel(False)
    ref = sta.forward_raster(q.cuda(), k.cuda(), v.cuda(), w.windows, w.text_len, w.has_text,
                             shape, w.tile)
    sta.device_status()
    assert (out.float() - ref.float()).abs().max().item() <= MAX_ABS
