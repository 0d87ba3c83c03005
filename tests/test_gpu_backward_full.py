"""GPU parity of the STA backward pass at the full video+text workload: the
bench's backward leg (B=1, 24 heads, d=128, (30,48,80) video + 256 text,
window (3,3,3), tile order).

dQ: sampled query rows (video rows of several tiles and text rows) of two
heads against the float64 oracle, row by row
(oracle.sta_bwd_oracle.sta_backward_query_rows), with the tolerance of the
small backward tests (max-abs <= 2e-2 max|ref|, mean-abs <= 1e-2 mean|ref|).

dK, dV: sampled key rows of two heads against the float64 oracle, element
by element (oracle.sta_bwd_oracle.sta_backward_key_rows, same tolerance):
rows of the text key block (valid and padded keys), of a corner video tile
(in the windows of the most query tiles once the window is shifted inward)
and of a mid-grid tile, and random video rows.  Also two identities of the
gradient, checked for every (batch, head) and column; they hold at any size,
so they cover every key row:
  sum over key rows of dV = sum over query rows of dO
      (dV = P^T dO and every row of P sums to one);
  sum over key rows of dK = 0
      (dK = dS^T q / sqrt(d) and every row of dS = P (dP - D) sums to zero,
       D_i being exactly sum_j P_ij dP_ij).
Tolerances: the dV sums within 0.5% of the column's random-walk scale
sqrt(sum_i dO_ic^2) (a key block left out, e.g. the text block with ~2% of
the attention mass, moves them by ~2%); the dK sums within 5% of
sqrt(sum_j dK_jc^2) (contributions left out make them of the order of that
scale times the square root of the fraction left out).
"""
import numpy as np
import pytest
import torch

import block_sparse_local_b200 as sta
from block_sparse_local_b200 import workloads
from oracle import sta_bwd_oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def full_backward():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    w = workloads.VIDEO_TEXT
    shape = (w.T, w.H, w.W)
    q, k, v = workloads.sta_inputs(w, device="cuda")            # raster order
    dout = workloads.randn_bf16(q.shape, 9191, device="cuda")
    qt, kt, vt, dot = (sta.tile_reorder(x, shape, w.tile, w.has_text) for x in (q, k, v, dout))
    ot, lse = sta.forward(qt, kt, vt, w.windows, w.text_len, w.has_text, shape, w.tile,
                          return_lse=True)
    dq, dk, dv = sta.backward(qt, kt, vt, ot, dot, lse, w.windows, w.text_len, w.has_text,
                              shape, w.tile)
    sta.device_status()
    dq_raster = sta.tile_unreorder(dq, shape, w.tile, w.has_text)
    dk_raster = sta.tile_unreorder(dk, shape, w.tile, w.has_text)
    dv_raster = sta.tile_unreorder(dv, shape, w.tile, w.has_text)
    sta.device_status()
    return w, (q, k, v, dout), dq_raster, dk, dv, dk_raster, dv_raster


def _tile_rows(w, tc, count, rng):
    """`count` raster rows of the video tile with tile coordinates tc."""
    ct, ch, cw = w.tile
    t = tc[0] * ct + rng.integers(0, ct, count)
    h = tc[1] * ch + rng.integers(0, ch, count)
    x = tc[2] * cw + rng.integers(0, cw, count)
    return (t * w.H + h) * w.W + x


def test_full_dq_sampled_rows(full_backward):
    w, (q, k, v, dout), dq = full_backward[:3]
    rng = np.random.default_rng(17)
    rows = np.unique(np.concatenate([rng.integers(0, w.L_v, size=48),
                                     np.arange(w.L_v, w.S, 16)]))
    for h in (0, 17):
        q64, k64, v64, do64 = (x[0, h].double().cpu().numpy() for x in (q, k, v, dout))
        ref = sta_bwd_oracle.sta_backward_query_rows(q64, k64, v64, do64, rows, w.T, w.H, w.W,
                                                     w.tile, tuple(w.windows[h]), w.text_len,
                                                     w.has_text)
        got = dq[0, h].float().cpu().numpy()[rows]
        err = np.abs(got - ref)
        assert err.max() <= 2e-2 * np.abs(ref).max(), (h, err.max(), np.abs(ref).max())
        assert err.mean() <= 1e-2 * np.abs(ref).mean(), (h, err.mean(), np.abs(ref).mean())


def test_full_dk_dv_sampled_key_rows(full_backward):
    w, (q, k, v, dout), _, _, _, dk, dv = full_backward
    rng = np.random.default_rng(23)
    text = w.L_v + np.array([0, 63, 127, 128, 199, 200, 255])   # 200.. are padding
    keys = np.unique(np.concatenate([text, _tile_rows(w, (0, 0, 0), 12, rng),
                                     _tile_rows(w, (2, 3, 5), 12, rng),
                                     rng.integers(0, w.L_v, 12)]))
    for h in (3, 20):
        q64, k64, v64, do64 = (x[0, h].double().cpu().numpy() for x in (q, k, v, dout))
        rk, rv = sta_bwd_oracle.sta_backward_key_rows(q64, k64, v64, do64, keys, w.T, w.H,
                                                      w.W, w.tile, tuple(w.windows[h]),
                                                      w.text_len, w.has_text)
        for name, got_all, ref in (("dk", dk, rk), ("dv", dv, rv)):
            got = got_all[0, h].float().cpu().numpy()[keys]
            err = np.abs(got - ref)
            assert err.max() <= 2e-2 * np.abs(ref).max(), (name, h, err.max())
            assert err.mean() <= 1e-2 * np.abs(ref).mean(), (name, h, err.mean())
            pad = keys >= w.L_v + w.text_len
            assert not got[pad].any(), (name, h)       # padded text keys: exactly zero


def test_full_dv_column_sums_equal_dout_column_sums(full_backward):
    w, (_, _, _, dout), _, _, dv = full_backward[:5]
    sdv = dv.double().sum(dim=2)                      # [B, heads, d]
    sdo = dout.double().sum(dim=2)
    scale = dout.double().pow(2).sum(dim=2).sqrt()
    ratio = ((sdv - sdo).abs() / scale).max().item()
    assert ratio <= 5e-3, ratio


def test_full_dk_column_sums_vanish(full_backward):
    dk = full_backward[3]
    sdk = dk.double().sum(dim=2)
    scale = dk.double().pow(2).sum(dim=2).sqrt()
    ratio = (sdk.abs() / scale).max().item()
    assert ratio <= 5e-2, ratio
