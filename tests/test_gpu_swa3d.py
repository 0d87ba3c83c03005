"""GPU parity of the token-level 3-D sliding-window kernel (mixed blocks)
against its float64 oracle; tolerance as for STA (max-abs <= 2e-2,
mean-abs <= 2e-3 per (batch, head))."""
import numpy as np
import pytest
import torch

import block_sparse_local_b200 as sta
from block_sparse_local_b200 import workloads
from oracle import swa3d_oracle

pytestmark = pytest.mark.gpu
MAX_ABS, MEAN_ABS = 2e-2, 2e-3


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    sta.lib()


def _check(w, window, rows=None, pairs=None, device="cpu"):
    q, k, v = workloads.sta_inputs(w, device=device)
    out = sta.swa3d_forward(q.cuda(), k.cuda(), v.cuda(), window, w.text_len, w.has_text,
                            (w.T, w.H, w.W), w.tile)
    sta.device_status()
    pairs = pairs or [(b, h) for b in range(w.B) for h in range(w.heads)]
    for b, h in pairs:
        q64, k64, v64 = (x[b, h].double().cpu().numpy() for x in (q, k, v))
        ref, _ = swa3d_oracle.swa3d_forward_rows(q64, k64, v64, w.T, w.H, w.W, window,
                                                 w.text_len, w.has_text, rows=rows)
        got = out[b, h].float().cpu().numpy()
        got = got if rows is None else got[rows]
        err = np.abs(got - ref)
        assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (b, h, err.max(), err.mean())


@pytest.mark.parametrize("shape,tile,window,text_len,has_text,d", [
    ((12, 16, 24), (6, 8, 8), (7, 9, 11), 0, False, 128),
    ((12, 16, 24), (6, 8, 8), (8, 10, 6), 200, True, 64),
    ((6, 24, 16), (2, 8, 8), (3, 5, 4), 37, True, 128),
    ((4, 16, 16), (2, 8, 8), (9, 40, 3), 256, True, 64),     # windows longer than the grid
    ((4, 16, 16), (2, 8, 8), (1, 1, 1), 0, False, 64),       # every query sees itself
])
def test_swa3d_matches_oracle(shape, tile, window, text_len, has_text, d):
    w = workloads.small_sta_case(*shape, tile, [(1, 1, 1)] * 2, text_len, has_text, d=d, seed=23)
    _check(w, window)


def test_swa3d_full_size_video_text_sampled():
    w = workloads.VIDEO_TEXT
    rng = np.random.default_rng(6)
    rows = np.unique(np.concatenate([np.arange(0, 384), rng.integers(0, w.L_v, 256),
                                     np.arange(w.L_v - 200, w.S)]))
    _check(w, (18, 24, 24), rows=rows, pairs=[(0, 0), (0, 23)], device="cuda")


def test_swa3d_rejects_unsupported_tiles():
    w = workloads.small_sta_case(1, 64, 64, (1, 16, 16), [(1, 1, 1)], 0, False, d=64, seed=1)
    q, k, v = workloads.sta_inputs(w)
    with pytest.raises(sta.StaError) as e:
        sta.swa3d_forward(q.cuda(), k.cuda(), v.cuda(), (1, 5, 5), 0, False, (1, 64, 64), w.tile)
    assert e.value.code == 2
