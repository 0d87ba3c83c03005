"""GPU parity of the fused STA attention against the float64 oracle, on sizes
the oracle finishes in seconds that still span several tiles, both slots of a
CTA, the leftover-block pairing and the ragged text tail.

Tolerance (bf16 inputs, fp32 accumulation, bf16 P and output):
max-abs <= 2e-2 and mean-abs <= 2e-3 per (batch, head).
"""
import numpy as np
import pytest
import torch

import block_sparse_local_b200 as sta
from block_sparse_local_b200 import workloads
from oracle import perm_oracle, sta_oracle

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 2e-2, 2e-3


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    sta.lib()


def _oracle(w, q, k, v, rows=None):
    q64, k64, v64 = (x.double().numpy() for x in (q, k, v))
    return sta_oracle.sta_forward_batched(q64, k64, v64, w.T, w.H, w.W, w.tile, w.windows,
                                          w.text_len, w.has_text, rows=rows)


def _compare(got, res, rows=None):
    for (b, h), (ref, _) in res.items():
        g = got[b, h] if rows is None else got[b, h][rows]
        err = np.abs(g - ref)
        assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (b, h, err.max(), err.mean())


def _run_tile_order(w, q, k, v, lse=False):
    """Oracle-side permutation on the CPU, GPU attention in tile order."""
    shape = (w.T, w.H, w.W)
    qt, kt, vt = (torch.from_numpy(perm_oracle.reorder(x.view(torch.int16).numpy(), *shape,
                                                       w.tile, w.has_text)).view(torch.bfloat16)
                  for x in (q, k, v))
    res = sta.forward(qt.cuda(), kt.cuda(), vt.cuda(), w.windows, w.text_len, w.has_text,
                      shape, w.tile, return_lse=lse)
    sta.device_status()
    o = res[0] if lse else res
    o = perm_oracle.unreorder(o.float().cpu().numpy(), *shape, w.tile, w.has_text)
    if lse:
        l = res[1].cpu().numpy()[..., None]
        l = perm_oracle.unreorder(l, *shape, w.tile, w.has_text)[..., 0]
        return o, l
    return o


CASES = [
    # (T,H,W), tile, windows, text_len, has_text, d, B
    ((18, 24, 32), (6, 8, 8), [(1, 3, 3)], 0, False, 64, 1),            # tiny workload
    ((12, 16, 24), (6, 8, 8), [(2, 2, 2), (1, 1, 3)], 200, True, 128, 1),
    ((12, 16, 24), (6, 8, 8), [(1, 2, 3)], 1, True, 128, 2),
    ((12, 16, 24), (6, 8, 8), [(2, 1, 2)], 128, True, 64, 1),
    ((12, 16, 24), (6, 8, 8), [(3, 3, 3)], 256, True, 128, 1),
    ((12, 16, 24), (6, 8, 8), [(1, 1, 1)], 0, True, 128, 1),             # text, no valid key
    ((1, 64, 64), (1, 16, 16), [(1, 3, 3), (1, 4, 2)], 0, False, 64, 2),  # 256-token tiles
    ((4, 24, 32), (2, 8, 8), [(1, 3, 3), (2, 2, 4)], 37, True, 128, 1),   # 128-token tiles
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0]}-{c[1]}-t{c[3]}-d{c[5]}")
def test_forward_matches_oracle(case):
    shape, tile, windows, text_len, has_text, d, B = case
    w = workloads.small_sta_case(*shape, tile, windows, text_len, has_text, d=d, B=B, seed=7)
    q, k, v = workloads.sta_inputs(w)
    got = _run_tile_order(w, q, k, v)
    _compare(got, _oracle(w, q, k, v))


def test_raster_api_matches_oracle():
    w = workloads.small_sta_case(4, 24, 32, (2, 8, 8), [(1, 3, 3), (2, 2, 4)], 37, True,
                                 d=128, seed=11)
    q, k, v = workloads.sta_inputs(w)
    out = sta.sliding_tile_attention(q.cuda(), k.cuda(), v.cuda(), w.windows, w.text_len,
                                     w.has_text, (w.T, w.H, w.W), w.tile)
    sta.device_status()
    _compare(out.float().cpu().numpy(), _oracle(w, q, k, v))


def test_lse_matches_oracle():
    w = workloads.small_sta_case(12, 16, 24, (6, 8, 8), [(2, 2, 2)], 100, True, d=128, seed=3)
    q, k, v = workloads.sta_inputs(w)
    out, lse = _run_tile_order(w, q, k, v, lse=True)
    res = _oracle(w, q, k, v)
    _compare(out, res)
    for (b, h), (_, ref_lse) in res.items():
        assert np.abs(lse[b, h] - ref_lse).max() < 1e-2


@pytest.mark.parametrize("d", [64, 128])
def test_constant_values_give_exact_ones(d):
    # softmax rows sum to one: with v = 1 every output is 1 (bf16 rounding of
    # the normalised sum), whatever the scores.
    w = workloads.small_sta_case(12, 16, 24, (6, 8, 8), [(2, 2, 3)], 77, True, d=d, seed=5)
    q, k, _ = workloads.sta_inputs(w)
    v = torch.ones_like(q)
    got = _run_tile_order(w, q, k, v)
    assert np.abs(got - 1.0).max() <= 2 ** -7


def test_full_window_is_dense_attention():
    # window covering the whole grid and every text key valid: plain attention
    w = workloads.small_sta_case(12, 16, 24, (6, 8, 8), [(9, 9, 9)], 256, True, d=64, seed=9)
    q, k, v = workloads.sta_inputs(w)
    got = _run_tile_order(w, q, k, v)
    ref = torch.nn.functional.scaled_dot_product_attention(q.double(), k.double(), v.double())
    err = np.abs(got - ref.numpy())
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS


RASTER_CASES = [
    # (T,H,W), tile, windows, text_len, has_text, d, B
    ((12, 16, 24), (6, 8, 8), [(2, 2, 2), (1, 1, 3)], 200, True, 128, 1),   # box 8x8x2
    ((1, 64, 64), (1, 16, 16), [(1, 3, 3)], 0, False, 64, 2),               # box 16x8x1
    ((4, 24, 32), (2, 8, 8), [(1, 3, 3), (2, 2, 4)], 37, True, 128, 1),      # 128-token tiles
    ((8, 32, 16), (2, 16, 8), [(3, 1, 2)], 129, True, 64, 1),               # box 8x16x1
    ((12, 16, 24), (6, 8, 8), [(1, 2, 3), (3, 1, 1), (1, 2, 3)], 5, True, 64, 2),  # B=2
]


@pytest.mark.parametrize("case", RASTER_CASES, ids=lambda c: f"{c[0]}-{c[1]}-t{c[3]}-d{c[5]}")
def test_fused_raster_forward_matches_oracle(case):
    shape, tile, windows, text_len, has_text, d, B = case
    w = workloads.small_sta_case(*shape, tile, windows, text_len, has_text, d=d, B=B, seed=17)
    q, k, v = workloads.sta_inputs(w)
    out, lse = sta.forward_raster(q.cuda(), k.cuda(), v.cuda(), w.windows, w.text_len,
                                  w.has_text, shape, w.tile, return_lse=True)
    sta.device_status()
    res = _oracle(w, q, k, v)
    _compare(out.float().cpu().numpy(), res)
    for (b, h), (_, ref_lse) in res.items():
        assert np.abs(lse[b, h].cpu().numpy() - ref_lse).max() < 1e-2


def test_non_box_tiles_fall_back_to_reorder_kernels():
    # 24 tokens along w do not divide a 128-row block: the fused raster path
    # refuses it and sliding_tile_attention uses the explicit permutation.
    w = workloads.small_sta_case(4, 4, 48, (4, 4, 24), [(1, 1, 2)], 0, False, d=64, seed=19)
    q, k, v = workloads.sta_inputs(w)
    with pytest.raises(sta.StaError) as err:
        sta.forward_raster(q.cuda(), k.cuda(), v.cuda(), w.windows, 0, False, (4, 4, 48), w.tile)
    assert err.value.code == 2
    out = sta.sliding_tile_attention(q.cuda(), k.cuda(), v.cuda(), w.windows, 0, False,
                                     (4, 4, 48), w.tile)
    sta.device_status()
    _compare(out.float().cpu().numpy(), _oracle(w, q, k, v))
