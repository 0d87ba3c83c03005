"""Plant plausible mistakes in the oracle (CPU only) and check a pin catches each.

Each mutation patches one oracle function for the duration of one test and
re-runs the pins of tests/test_oracle.py that should fail.
"""
import numpy as np
import pytest

import oracle.geometry as geometry
import oracle.sta_oracle as sta_oracle
import oracle.tiles_oracle as tiles_oracle
import oracle.swa_oracle as swa_oracle
from tests import test_oracle as pins


def _unclamped_start(c, w, n):
    we = min(w, n)
    return c - we // 2, we


def _start_no_clip(c, w, n):
    s = min(max(c - w // 2, 0), max(n - w, 0))
    return s, w


def _start_off_by_one(c, w, n):
    we = min(w, n)
    return min(max(c - (we - 1) // 2 - 1, 0), n - we), we


@pytest.mark.parametrize("bad", [_unclamped_start, _start_no_clip, _start_off_by_one])
def test_window_start_mistakes_are_caught(monkeypatch, golden_dir, bad):
    for mod in (geometry, sta_oracle, tiles_oracle):
        monkeypatch.setattr(mod, "window_start", bad)
    failures = 0
    for pin in (lambda: pins.test_window_starts_demo(golden_dir),
                lambda: pins.test_tile_lists_demo_10x10(golden_dir),
                lambda: pins.test_tile_lists_tiny(golden_dir),
                pins.test_tile_list_counts_2d_and_clip,
                lambda: pins.test_form_a_matches_form_b(pins.SMALL_CASES[4])):
        try:
            pin()
        except (AssertionError, IndexError, ValueError):
            failures += 1
    assert failures > 0


def test_wrong_scale_is_caught(monkeypatch):
    orig = sta_oracle.sta_forward_rows

    def bad(q, k, v, *a, **kw):   # scale 1/d instead of 1/sqrt(d)
        return orig(q / np.sqrt(q.shape[1]), k, v, *a, **kw)

    monkeypatch.setattr(sta_oracle, "sta_forward_rows", bad)
    with pytest.raises(AssertionError):
        pins.test_full_window_is_dense_attention(0, False)


def test_dropped_text_keys_are_caught(monkeypatch):
    orig = sta_oracle.allowed_keys

    def bad(qrow, T, H, W, tile, window, text_len, has_text):
        keys = orig(qrow, T, H, W, tile, window, text_len, has_text)
        return keys[keys < T * H * W]

    monkeypatch.setattr(sta_oracle, "allowed_keys", bad)
    with pytest.raises(AssertionError):
        pins.test_full_window_is_dense_attention(100, True)


def test_transposed_tile_coordinates_are_caught(monkeypatch):
    import oracle.perm_oracle as perm_oracle

    def bad(T, H, W, tile):   # h and w swapped inside the tile
        ct, ch, cw = tile
        NT, NH, NW = geometry.tile_grid(T, H, W, tile)
        r = np.arange(T * H * W)
        t, h, w = r // (H * W), (r // W) % H, r % W
        tid = ((t // ct) * NH + h // ch) * NW + w // cw
        inn = ((t % ct) * cw + w % cw) * ch + h % ch
        return tid * (ct * ch * cw) + inn

    monkeypatch.setattr(perm_oracle, "tile_position_of_raster", bad)
    with pytest.raises(AssertionError):
        pins.test_permutation_formula_is_tile_transpose(4, 6, 6, (2, 3, 2))


def test_swa_off_by_one_window_is_caught(monkeypatch):
    def bad(i, S, window, causal):
        return np.arange(max(0, i - window), i + 1)

    monkeypatch.setattr(swa_oracle, "swa_allowed", bad)
    with pytest.raises(AssertionError):
        pins.test_swa_band_matches_brute_force_mask()
