"""GPU parity of the Hilbert-order path: the permutation and the block lists
are bit-exact against the oracle; block-sparse slide attention matches the
float64 oracle (max-abs <= 2e-2, mean-abs <= 2e-3 per (batch, head))."""
import numpy as np
import pytest
import torch

import block_sparse_local_b200 as sta
from block_sparse_local_b200 import workloads
from oracle import hilbert_oracle as ho
from oracle import swa3d_oracle

pytestmark = pytest.mark.gpu
MAX_ABS, MEAN_ABS = 2e-2, 2e-3


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    sta.lib()


@pytest.mark.parametrize("n,d", [(16, 64), (64, 128), (256, 64)])
def test_hilbert_reorder_bit_exact(n, d):
    x = torch.randint(-32768, 32767, (2, 3, n * n, d), dtype=torch.int16)
    y = sta.hilbert_reorder(x.view(torch.bfloat16).cuda(), n, True)
    want = x.numpy()[:, :, ho.hilbert_order(n), :]
    assert np.array_equal(y.view(torch.int16).cpu().numpy(), want)
    z = sta.hilbert_reorder(y, n, False)
    sta.device_status()
    assert torch.equal(z.view(torch.int16).cpu(), x)


@pytest.mark.parametrize("n,w,order", [(64, 9, "hilbert"), (64, 40, "hilbert"),
                                       (128, 5, "raster"), (128, 13, "hilbert"),
                                       (256, 21, "raster"), (256, 21, "hilbert")])
def test_block_lists_bit_exact(n, w, order):
    o = ho.hilbert_order(n) if order == "hilbert" else ho.raster_order(n)
    cls = ho.block_classes(n, w, o) if n <= 64 else ho.block_classes_rect(n, w, o)
    counts, ids, kcls = sta.build_slide_block_lists(n, w, order)
    sta.device_status()
    counts, ids, kcls = counts.cpu().numpy(), ids.cpu().numpy(), kcls.cpu().numpy()
    for qb in range(cls.shape[0]):
        want = np.nonzero(cls[qb])[0]
        assert counts[qb] == len(want)
        assert np.array_equal(ids[qb, :len(want)], want)
        assert np.array_equal(kcls[qb, :len(want)], cls[qb, want])
        assert (ids[qb, len(want):] == -1).all()


@pytest.mark.parametrize("n,w,order,d", [(32, 5, "hilbert", 64), (32, 9, "hilbert", 128),
                                         (128, 9, "raster", 128), (128, 9, "hilbert", 64)])
def test_slide2d_matches_oracle(n, w, order, d):
    wl = workloads.small_sta_case(1, n, n, (1, n, n), [(1, 1, 1)] * 2, 0, False, d=d, seed=31)
    q, k, v = workloads.sta_inputs(wl)
    out = sta.slide_attention_2d(q.cuda(), k.cuda(), v.cuda(), n, w, order)
    sta.device_status()
    rows = np.arange(n * n) if n <= 32 else np.unique(
        np.concatenate([np.arange(0, 300), np.random.default_rng(2).integers(0, n * n, 400)]))
    for h in range(2):
        q64, k64, v64 = (x[0, h].double().numpy() for x in (q, k, v))
        ref, _ = swa3d_oracle.swa3d_forward_rows(q64, k64, v64, 1, n, n, (1, w, w), 0, False,
                                                 rows=rows)
        err = np.abs(out[0, h].float().cpu().numpy()[rows] - ref)
        assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (h, err.max(), err.mean())


def test_slide2d_full_size_sampled():
    n, w = 256, 21
    wl = workloads.small_sta_case(1, n, n, (1, 16, 16), [(1, 1, 1)] * 4, 0, False, d=64, B=2,
                                  seed=33)
    q, k, v = workloads.sta_inputs(wl, device="cuda")
    out = sta.slide_attention_2d(q, k, v, n, w, "hilbert")
    sta.device_status()
    rows = np.unique(np.random.default_rng(3).integers(0, n * n, 300))
    for b, h in [(0, 0), (1, 3)]:
        q64, k64, v64 = (x[b, h].double().cpu().numpy() for x in (q, k, v))
        ref, _ = swa3d_oracle.swa3d_forward_rows(q64, k64, v64, 1, n, n, (1, w, w), 0, False,
                                                 rows=rows)
        err = np.abs(out[b, h].float().cpu().numpy()[rows] - ref)
        assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS
