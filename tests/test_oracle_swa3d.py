"""Pins of the token-level 3-D sliding-window oracle (the mixed-block baseline)."""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import sta_oracle, swa3d_oracle


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


@pytest.mark.parametrize("T,H,W,window,text_len,has_text", [
    (4, 6, 5, (3, 3, 3), 0, False),
    (3, 6, 8, (2, 4, 3), 37, True),
    (5, 4, 6, (9, 2, 4), 256, True),
])
def test_equals_sta_with_single_token_tiles(T, H, W, window, text_len, has_text):
    # with tiles of one token a window of tiles is a window of tokens
    S = T * H * W + (256 if has_text else 0)
    q, k, v = (_rand((S, 8), s) for s in (1, 2, 3))
    a, la = swa3d_oracle.swa3d_forward_rows(q, k, v, T, H, W, window, text_len, has_text)
    b, lb = sta_oracle.sta_forward_rows(q, k, v, T, H, W, (1, 1, 1), window, text_len, has_text)
    np.testing.assert_allclose(a, b, atol=1e-12)
    np.testing.assert_allclose(la, lb, atol=1e-12)


def test_mask_form_matches_row_form():
    T, H, W, window, text_len = 4, 6, 6, (3, 4, 2), 11
    S = T * H * W + 256
    q, k, v = (_rand((S, 8), s) for s in (4, 5, 6))
    mask = swa3d_oracle.swa3d_mask(T, H, W, window, text_len, True)
    ref, _, _ = sta_oracle.masked_softmax_attention(q, k, v, mask, 1 / np.sqrt(8))
    got, _ = swa3d_oracle.swa3d_forward_rows(q, k, v, T, H, W, window, text_len, True)
    np.testing.assert_allclose(got, ref, atol=1e-12)


def test_full_and_unit_windows():
    T, H, W = 3, 4, 5
    S = T * H * W
    q, k, v = (_rand((S, 8), s) for s in (7, 8, 9))
    full, _ = swa3d_oracle.swa3d_forward_rows(q, k, v, T, H, W, (3, 4, 5), 0, False)
    ref = F.scaled_dot_product_attention(*(torch.from_numpy(x) for x in (q, k, v))).numpy()
    np.testing.assert_allclose(full, ref, atol=1e-12)
    unit, _ = swa3d_oracle.swa3d_forward_rows(q, k, v, T, H, W, (1, 1, 1), 0, False)
    np.testing.assert_allclose(unit, v, atol=1e-12)


def test_every_query_sees_a_full_window_around_itself():
    T, H, W, window = 30, 48, 80, (18, 24, 24)
    rng = np.random.default_rng(0)
    for r in list(rng.integers(0, T * H * W, 30)) + [0, T * H * W - 1]:
        keys = swa3d_oracle.allowed_keys(int(r), T, H, W, window, 0, False)
        assert len(keys) == 18 * 24 * 24
        t, h, w = keys // (H * W), (keys // W) % H, keys % W
        assert [t.max() - t.min() + 1, h.max() - h.min() + 1, w.max() - w.min() + 1] == [18, 24, 24]
        qt, qh, qw = r // (H * W), (r // W) % H, r % W
        assert t.min() <= qt <= t.max() and h.min() <= qh <= h.max() and w.min() <= qw <= w.max()


def test_retained_pairs_closed_form():
    # same per-query key count as STA (3,3,3) tiles on (30,48,80): 18*24*24 + text
    got = swa3d_oracle.swa3d_retained_pairs(30, 48, 80, (18, 24, 24), 200, True)
    assert got == sta_oracle.retained_pairs(30, 48, 80, (6, 8, 8), (3, 3, 3), 200, True)


def test_off_by_one_start_is_caught(monkeypatch):
    def bad(x, w, n):
        we = min(w, n)
        return min(max(x - we // 2 + 1, 0), n - we), we
    monkeypatch.setattr(swa3d_oracle, "token_window_start", bad)
    with pytest.raises(AssertionError):
        test_equals_sta_with_single_token_tiles(4, 6, 5, (3, 3, 3), 0, False)
