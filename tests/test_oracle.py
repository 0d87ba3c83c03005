"""Pins of the CPU oracle against what the STA README and mathematics fix.

No test here compares the oracle with itself: each check is a hand-derived
fixture from the page (tests/golden), a closed form, a special case that
reduces to a library routine (torch's scaled_dot_product_attention in
float64), or brute force on tiny inputs.
"""
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import geometry, perm_oracle, sta_oracle, swa_oracle, tiles_oracle


def _read_lists(path):
    starts, lists, extra = None, {}, {}
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if ":" in line:
                key, vals = line.split(":")
                lists[tuple(int(x) for x in key.split())] = [int(x) for x in vals.split()]
            else:
                parts = line.split()
                extra[parts[0]] = [int(x) for x in parts[1:]]
    return lists, extra


def _sdpa64(q, k, v, mask=None, causal=False):
    """Library attention in float64: q,k,v numpy [S,d] (or [H,S,d])."""
    tq, tk, tv = (torch.from_numpy(np.ascontiguousarray(x)) for x in (q, k, v))
    m = None if mask is None else torch.from_numpy(mask)
    return F.scaled_dot_product_attention(tq, tk, tv, attn_mask=m,
                                          is_causal=causal).numpy()


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# --------------------------------------------------------------------------
# window geometry and tile lists: hand-derived fixtures from the page
# --------------------------------------------------------------------------
def test_window_starts_demo(golden_dir):
    _, extra = _read_lists(os.path.join(golden_dir, "demo_10x10_tile_lists.txt"))
    got = [geometry.window_start(c, 3, 5)[0] for c in range(5)]
    assert got == extra["starts"]


def test_tile_lists_demo_10x10(golden_dir):
    lists, extra = _read_lists(os.path.join(golden_dir, "demo_10x10_tile_lists.txt"))
    counts, ids = tiles_oracle.kv_tile_lists(1, 10, 10, (1, 2, 2), [(1, 3, 3)], 0, False)
    assert counts.shape == (1, 25)
    for (r, c), want in lists.items():
        q = r * 5 + c
        assert ids[0, q, :counts[0, q]].tolist() == want, (r, c)
    # every query token sees a full 6x6 window
    for row in range(100):
        keys = sta_oracle.allowed_keys(row, 1, 10, 10, (1, 2, 2), (1, 3, 3), 0, False)
        assert len(keys) == extra["tokens_per_query"][0]


def test_tile_lists_tiny(golden_dir):
    lists, _ = _read_lists(os.path.join(golden_dir, "tiny_tile_lists.txt"))
    counts, ids = tiles_oracle.kv_tile_lists(18, 24, 32, (6, 8, 8), [(1, 3, 3)], 0, False)
    assert counts.shape == (1, 36)
    assert (counts == 9).all()
    for (t, h, w), want in lists.items():
        q = (t * 3 + h) * 4 + w
        assert ids[0, q, :9].tolist() == want, (t, h, w)


def test_usage_window_extent(golden_dir):
    _, g = _read_lists(os.path.join(golden_dir, "usage_window_extent.txt"))
    T, H, W = g["grid"]
    tile, window = tuple(g["tile"]), tuple(g["window"])
    rng = np.random.default_rng(0)
    for row in list(rng.integers(0, T * H * W, size=40)) + [0, T * H * W - 1]:
        keys = sta_oracle.allowed_keys(int(row), T, H, W, tile, window, 0, False)
        assert len(keys) == g["video_keys_per_query"][0]
        t, h, w = keys // (H * W), (keys // W) % H, keys % W
        ext = [t.max() - t.min() + 1, h.max() - h.min() + 1, w.max() - w.min() + 1]
        assert ext == g["extent"]
        qt, qh, qw = row // (H * W), (row // W) % H, row % W
        assert t.min() <= qt <= t.max() and h.min() <= qh <= h.max() and w.min() <= qw <= w.max()


def test_tile_list_counts_video_text_geometry():
    # (30,48,80)/(6,8,8) = (5,6,10) tiles, window (3,3,3), 200 valid text keys
    counts, ids = tiles_oracle.kv_tile_lists(30, 48, 80, (6, 8, 8), [(3, 3, 3)], 200, True)
    assert counts.shape == (1, 301)
    assert (counts[0, :300] == 28).all()          # 27 tiles + the text block
    assert (ids[0, :300, 27] == 300).all()
    assert counts[0, 300] == 301                  # text queries: all tiles + text
    assert ids[0, 300, :301].tolist() == list(range(301))
    # without valid text keys the sentinel disappears
    c0, _ = tiles_oracle.kv_tile_lists(30, 48, 80, (6, 8, 8), [(3, 3, 3)], 0, True)
    assert (c0[0, :300] == 27).all() and c0[0, 300] == 300


def test_tile_list_counts_2d_and_clip():
    c, _ = tiles_oracle.kv_tile_lists(1, 256, 256, (1, 16, 16), [(1, 5, 5)], 0, False)
    assert (c == 25).all()
    c, _ = tiles_oracle.kv_tile_lists(1, 256, 256, (1, 16, 16), [(1, 16, 16)], 0, False)
    assert (c == 256).all()
    c, _ = tiles_oracle.kv_tile_lists(1, 64, 64, (1, 16, 16), [(3, 9, 9)], 0, False)
    assert (c == 16).all()    # windows longer than the grid clip to it


def test_retained_pairs_closed_form():
    # per head of the video+text workload, counted by hand:
    # 300 tiles * 27 tiles * 384^2 + 115200*200 + 256*(115200+200)
    want = 300 * 27 * 384 * 384 + 115200 * 200 + 256 * (115200 + 200)
    assert want == 1246976000
    got = sta_oracle.retained_pairs(30, 48, 80, (6, 8, 8), (3, 3, 3), 200, True)
    assert got == want


# --------------------------------------------------------------------------
# attention values
# --------------------------------------------------------------------------
SMALL_CASES = [
    # T, H, W, tile, window, text_len, has_text
    (4, 4, 6, (2, 2, 2), (1, 1, 3), 0, False),
    (4, 4, 6, (2, 2, 2), (2, 2, 2), 37, True),    # even windows
    (6, 4, 4, (2, 2, 2), (3, 1, 2), 1, True),
    (2, 6, 8, (1, 2, 2), (1, 3, 3), 256, True),
    (2, 6, 8, (1, 2, 2), (5, 9, 2), 0, True),     # windows longer than the grid
    (1, 10, 10, (1, 2, 2), (1, 3, 3), 0, False),  # the README's 2-D demo
]


@pytest.mark.parametrize("case", SMALL_CASES)
def test_form_a_matches_form_b(case):
    T, H, W, tile, window, text_len, has_text = case
    S = geometry.seq_len(T, H, W, has_text)
    q, k, v = (_rand((S, 16), s) for s in (1, 2, 3))
    out_a, lse_a = sta_oracle.sta_forward_dense(q, k, v, T, H, W, tile, window, text_len, has_text)
    out_b, lse_b = sta_oracle.sta_forward_rows(q, k, v, T, H, W, tile, window, text_len, has_text)
    np.testing.assert_allclose(out_a, out_b, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse_a, lse_b, rtol=0, atol=1e-12)


@pytest.mark.parametrize("text_len,has_text", [(0, False), (256, True), (100, True), (0, True)])
def test_full_window_is_dense_attention(text_len, has_text):
    T, H, W, tile = 4, 6, 8, (2, 2, 2)
    S = geometry.seq_len(T, H, W, has_text)
    q, k, v = (_rand((S, 32), s) for s in (4, 5, 6))
    out, _ = sta_oracle.sta_forward_rows(q, k, v, T, H, W, tile, (2, 3, 4), text_len, has_text)
    mask = None
    if has_text and text_len < 256:
        mask = np.ones((S, S), dtype=bool)
        mask[:, T * H * W + text_len:] = False   # key padding only
    ref = _sdpa64(q, k, v, mask)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_unit_window_is_block_diagonal():
    T, H, W, tile = 4, 6, 8, (2, 3, 4)
    ct, ch, cw = tile
    S = T * H * W
    q, k, v = (_rand((S, 16), s) for s in (7, 8, 9))
    out, _ = sta_oracle.sta_forward_rows(q, k, v, T, H, W, tile, (1, 1, 1), 0, False)

    def tiles(x):  # [S,d] raster -> [ntiles, V, d] via reshape/transpose
        d = x.shape[1]
        x = x.reshape(T // ct, ct, H // ch, ch, W // cw, cw, d)
        return x.transpose(0, 2, 4, 1, 3, 5, 6).reshape(-1, ct * ch * cw, d)

    ref = _sdpa64(tiles(q), tiles(k), tiles(v))
    np.testing.assert_allclose(tiles(out), ref, rtol=0, atol=1e-12)


def test_rows_sum_to_one_and_constant_values():
    T, H, W, tile, window = 4, 4, 6, (2, 2, 2), (1, 2, 3)
    S = geometry.seq_len(T, H, W, True)
    q, k = _rand((S, 8), 10), _rand((S, 8), 11)
    mask = sta_oracle.sta_mask(T, H, W, tile, window, 50, True)
    _, _, p = sta_oracle.masked_softmax_attention(q, k, np.ones((S, 8)), mask, 0.5)
    assert np.abs(p.sum(1) - 1).max() < 1e-12
    out, _ = sta_oracle.sta_forward_rows(q, k, np.ones((S, 8)), T, H, W, tile, window, 50, True)
    assert np.abs(out - 1).max() < 1e-12


def test_zero_query_gives_mean_and_log_count():
    # q = 0: every allowed score is 0, so out = mean of the allowed values and
    # lse = ln(#allowed keys); the count per video query is the full window of
    # tiles times the tile volume plus the valid text keys.
    T, H, W, tile, window, text_len = 6, 4, 8, (2, 2, 2), (3, 1, 3), 19
    S = geometry.seq_len(T, H, W, True)
    v = _rand((S, 8), 12)
    k = _rand((S, 8), 13)
    out, lse = sta_oracle.sta_forward_rows(np.zeros((S, 8)), k, v, T, H, W, tile, window,
                                           text_len, True)
    Lv = T * H * W
    nvid = 3 * 1 * 3 * 8
    assert np.allclose(lse[:Lv], np.log(nvid + text_len), atol=1e-12)
    assert np.allclose(lse[Lv:], np.log(Lv + text_len), atol=1e-12)
    np.testing.assert_allclose(out[Lv:], np.broadcast_to(
        np.concatenate([v[:Lv], v[Lv:Lv + text_len]]).mean(0), (S - Lv, 8)), atol=1e-12)


def test_batched_per_head_windows():
    T, H, W, tile = 4, 4, 4, (2, 2, 2)
    windows = [(1, 1, 1), (2, 2, 2)]
    S = T * H * W
    q, k, v = (_rand((2, 2, S, 8), s) for s in (14, 15, 16))
    res = sta_oracle.sta_forward_batched(q, k, v, T, H, W, tile, windows, 0, False)
    # head 1's window covers the whole grid: dense attention
    ref = _sdpa64(q[1, 1], k[1, 1], v[1, 1])
    np.testing.assert_allclose(res[(1, 1)][0], ref, atol=1e-12)
    # head 0 differs from dense
    assert np.abs(res[(0, 0)][0] - _sdpa64(q[0, 0], k[0, 0], v[0, 0])).max() > 1e-3


# --------------------------------------------------------------------------
# permutation
# --------------------------------------------------------------------------
@pytest.mark.parametrize("T,H,W,tile", [(18, 24, 32, (6, 8, 8)), (1, 32, 48, (1, 16, 16)),
                                        (4, 6, 6, (2, 3, 2))])
def test_permutation_formula_is_tile_transpose(T, H, W, tile):
    ct, ch, cw = tile
    p = perm_oracle.tile_position_of_raster(T, H, W, tile)
    # textbook identity: tile order = raster ids reshaped into tiles
    ids = np.arange(T * H * W).reshape(T // ct, ct, H // ch, ch, W // cw, cw)
    tile_order = ids.transpose(0, 2, 4, 1, 3, 5).reshape(-1)   # raster id at tile pos
    inv = np.empty_like(tile_order)
    inv[tile_order] = np.arange(tile_order.size)
    assert (p == inv).all()


def test_reorder_roundtrip_and_text_rows():
    T, H, W, tile = 4, 6, 4, (2, 3, 2)
    S = T * H * W + 256
    x = _rand((2, 3, S, 4), 17)
    y = perm_oracle.reorder(x, T, H, W, tile, True)
    assert (y[..., T * H * W:, :] == x[..., T * H * W:, :]).all()
    assert (perm_oracle.unreorder(y, T, H, W, tile, True) == x).all()
    assert not (y == x).all()


# --------------------------------------------------------------------------
# token-level sliding window with GQA
# --------------------------------------------------------------------------
def test_swa_long_window_is_causal_attention():
    S, d = 40, 8
    q, k, v = _rand((4, S, d), 18), _rand((2, S, d), 19), _rand((2, S, d), 20)
    res = swa_oracle.swa_forward(q, k, v, window=S + 3, causal=True)
    kk = np.repeat(k, 2, axis=0)
    vv = np.repeat(v, 2, axis=0)
    ref = _sdpa64(q, kk, vv, causal=True)
    for h in range(4):
        np.testing.assert_allclose(res[h][0], ref[h], atol=1e-12)


def test_swa_unit_window_returns_values():
    S, d = 17, 8
    q, k, v = _rand((2, S, d), 21), _rand((1, S, d), 22), _rand((1, S, d), 23)
    res = swa_oracle.swa_forward(q, k, v, window=1, causal=True)
    for h in range(2):
        np.testing.assert_allclose(res[h][0], v[0], atol=1e-12)


def test_swa_band_matches_brute_force_mask():
    S, d, w = 30, 8, 7
    q, k, v = _rand((1, S, d), 24), _rand((1, S, d), 25), _rand((1, S, d), 26)
    i = np.arange(S)[:, None]
    j = np.arange(S)[None, :]
    for causal, band in ((True, (j <= i) & (j > i - w)), (False, np.abs(i - j) < w)):
        res = swa_oracle.swa_forward(q, k, v, window=w, causal=causal)
        ref = _sdpa64(q[0], k[0], v[0], mask=band)
        np.testing.assert_allclose(res[0][0], ref, atol=1e-12)


def test_swa_pair_count_closed_form():
    S, w = 32768, 4096
    want = w * (w + 1) // 2 + (S - w) * w
    assert swa_oracle.swa_retained_pairs(S, w) == want == 125831168
