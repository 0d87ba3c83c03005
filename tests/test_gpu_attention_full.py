"""GPU parity at the full workload sizes, in the launch configuration bench.py
times (raster API: reorder -> tile lists + fused attention -> unreorder).

The oracle computes sampled rows one query tile at a time: for each checked
(batch, head), every row of the first, a middle and the last video query
tile, 256 seeded random video rows, and (with text) all 256 text rows.
Inputs are drawn on the GPU from seeded generators and copied back for the
oracle.
"""
import numpy as np
import pytest
import torch

import block_sparse_local_b200 as sta
from block_sparse_local_b200 import workloads
from oracle import sta_oracle, swa_oracle

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 2e-2, 2e-3


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    sta.lib()


def _tile_rows(w, tq):
    ct, ch, cw = w.tile
    NH, NW = w.H // ch, w.W // cw
    qt, qh, qw = tq // (NH * NW), (tq // NW) % NH, tq % NW
    tt = np.arange(qt * ct, (qt + 1) * ct)
    hh = np.arange(qh * ch, (qh + 1) * ch)
    ww = np.arange(qw * cw, (qw + 1) * cw)
    return ((tt[:, None, None] * w.H + hh[None, :, None]) * w.W + ww[None, None, :]).ravel()


def _sample_rows(w, seed):
    NV = (w.T // w.tile[0]) * (w.H // w.tile[1]) * (w.W // w.tile[2])
    rng = np.random.default_rng(seed)
    rows = [_tile_rows(w, 0), _tile_rows(w, NV // 2 + 1), _tile_rows(w, NV - 1),
            rng.integers(0, w.L_v, size=256)]
    if w.has_text:
        rows.append(np.arange(w.L_v, w.S))
    return np.unique(np.concatenate(rows))


def _check(w, pairs, seed=0):
    q, k, v = workloads.sta_inputs(w, device="cuda")
    out = sta.sliding_tile_attention(q, k, v, w.windows, w.text_len, w.has_text,
                                     (w.T, w.H, w.W), w.tile)
    sta.device_status()
    rows = _sample_rows(w, seed)
    for b, h in pairs:
        q64, k64, v64 = (x[b, h].double().cpu().numpy() for x in (q, k, v))
        ref, _ = sta_oracle.sta_forward_rows(q64, k64, v64, w.T, w.H, w.W, w.tile,
                                             tuple(w.windows[h]), w.text_len, w.has_text,
                                             rows=rows)
        got = out[b, h].float().cpu().numpy()[rows]
        err = np.abs(got - ref)
        assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (b, h, err.max(), err.mean())
    assert torch.isfinite(out.float()).all()
    return out


def test_video_text_full_size():
    w = workloads.VIDEO_TEXT
    _check(w, [(0, 0), (0, 11), (0, 23)])


def test_video_only_per_head_windows_full_size():
    w = workloads.VIDEO_ONLY
    # one head of every window class, both batch elements
    firsts = {}
    for h, win in enumerate(w.windows):
        firsts.setdefault(win, h)
    pairs = [(b, h) for b in (0, 1) for h in sorted(firsts.values())]
    _check(w, pairs, seed=1)


def test_image_2d_full_size():
    _check(workloads.IMAGE_2D, [(0, 0), (7, 15)], seed=2)


def test_image_2d_full_window_equals_dense():
    w = workloads.IMAGE_2D_FULL
    out = _check(w, [(3, 5)], seed=3)
    # and against the library dense attention on the GPU for one batch item
    q, k, v = workloads.sta_inputs(w, device="cuda")
    ref = torch.nn.functional.scaled_dot_product_attention(q[:1].float(), k[:1].float(),
                                                           v[:1].float())
    err = (out[:1].float() - ref).abs()
    assert err.max().item() <= MAX_ABS and err.mean().item() <= MEAN_ABS


# ------------------------------------------------------------------ sliding window
SWA_SMALL = [
    # B, hq, hkv, d, S, window
    (1, 4, 2, 128, 1024, 300),
    (2, 6, 2, 64, 768, 128),      # group of 3: one single-slot item per group
    (1, 2, 2, 128, 512, 1),
    (1, 4, 1, 64, 640, 5000),     # window longer than the sequence: causal attention
]


@pytest.mark.parametrize("B,hq,hkv,d,S,window", SWA_SMALL)
def test_swa_matches_oracle(B, hq, hkv, d, S, window):
    w = workloads.SwaWorkload("swa_small", B, hq, hkv, d, S, window, True, 1.0, 13)
    q, k, v = workloads.swa_inputs(w)
    out = sta.swa_forward(q.cuda(), k.cuda(), v.cuda(), window).float().cpu().numpy()
    sta.device_status()
    for b in range(B):
        res = swa_oracle.swa_forward(q[b].double().numpy(), k[b].double().numpy(),
                                     v[b].double().numpy(), window, True)
        for h, (ref, _) in res.items():
            err = np.abs(out[b, h] - ref)
            assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (b, h, err.max())


def test_swa_full_size_sampled():
    w = workloads.SWA_GQA
    q, k, v = workloads.swa_inputs(w, device="cuda")
    out = sta.swa_forward(q, k, v, w.window)
    sta.device_status()
    rng = np.random.default_rng(4)
    rows = np.unique(np.concatenate([np.arange(0, 300), np.arange(4000, 4200),
                                     rng.integers(0, w.S, 200), np.arange(w.S - 130, w.S)]))
    heads = [0, 5, 31]
    res = swa_oracle.swa_forward(q[0].double().cpu().numpy(), k[0].double().cpu().numpy(),
                                 v[0].double().cpu().numpy(), w.window, True, rows=rows,
                                 heads=heads)
    for h in heads:
        err = np.abs(out[0, h].float().cpu().numpy()[rows] - res[h][0])
        assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (h, err.max())
