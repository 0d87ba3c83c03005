"""Token-level 3-D sliding-window attention on the video grid (oracle side).

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

This is the "2D/3D Sliding Window Attention" that the STA README's section
"Why is STA Fast?" compares STA against: every query token has its own window
of keys, so the tile-by-tile blocks of the attention map are mostly mixed
(partly masked).  Reading taken (the page gives no formula): the window is
counted in tokens, (Wt, Wh, Ww), centred on the query token and shifted
inward at the grid border so that it always spans the full window (the same
border rule as STA's window of tiles, at token granularity, as in
neighbourhood attention); text tokens follow STA's rules (video queries also
see the first text_len text keys; text queries see every video key and the
first text_len text keys).

out_i = softmax over allowed j of (q_i . k_j / sqrt(d)), times v_j; float64.
"""
import numpy as np

from .geometry import TEXT_PAD


def token_window_start(x, w, n):
    """First token and extent of the window along one axis (centred, clamped)."""
    we = min(w, n)
    s = x - we // 2
    if s < 0:
        s = 0
    if s > n - we:
        s = n - we
    return s, we


def allowed_keys(qrow, T, H, W, window, text_len, has_text):
    """Sorted raster indices of the keys that query ``qrow`` may attend to."""
    Lv = T * H * W
    if qrow >= Lv:
        return np.arange(Lv + text_len)
    t, h, w = qrow // (H * W), (qrow // W) % H, qrow % W
    (st, et), (sh, eh), (sw, ew) = (token_window_start(t, window[0], T),
                                    token_window_start(h, window[1], H),
                                    token_window_start(w, window[2], W))
    tt = np.arange(st, st + et)
    hh = np.arange(sh, sh + eh)
    ww = np.arange(sw, sw + ew)
    keys = ((tt[:, None, None] * H + hh[None, :, None]) * W + ww[None, None, :]).reshape(-1)
    if has_text and text_len > 0:
        keys = np.concatenate([keys, Lv + np.arange(text_len)])
    return keys


def swa3d_forward_rows(q, k, v, T, H, W, window, text_len, has_text, rows=None):
    """q, k, v: float64 [S, d] raster order of one (batch, head).

    Returns (out [len(rows), d], lse [len(rows)]), one gather + matmul per row.
    """
    S, d = q.shape
    Lv = T * H * W
    if S != Lv + (TEXT_PAD if has_text else 0):
        raise ValueError("sequence length does not match the grid")
    scale = 1.0 / np.sqrt(d)
    rows = np.arange(S) if rows is None else np.asarray(rows, dtype=np.int64)
    out = np.empty((len(rows), d))
    lse = np.empty(len(rows))
    for pos, r in enumerate(rows):
        keys = allowed_keys(int(r), T, H, W, window, text_len, has_text)
        s = (k[keys] @ q[r]) * scale
        m = s.max()
        p = np.exp(s - m)
        l = p.sum()
        out[pos] = (p @ v[keys]) / l
        lse[pos] = m + np.log(l)
    return out, lse


def swa3d_mask(T, H, W, window, text_len, has_text):
    """Explicit S x S boolean mask (tiny grids), by brute force over coordinates."""
    Lv = T * H * W
    S = Lv + (TEXT_PAD if has_text else 0)
    r = np.arange(Lv)
    coords = (r // (H * W), (r // W) % H, r % W)
    dims = (T, H, W)
    mask = np.zeros((S, S), dtype=bool)
    ok = np.ones((Lv, Lv), dtype=bool)
    for a in range(3):
        se = [token_window_start(int(x), window[a], dims[a]) for x in coords[a]]
        lo = np.array([s for s, _ in se])
        hi = lo + np.array([e for _, e in se])
        kc = coords[a][None, :]
        ok &= (kc >= lo[:, None]) & (kc < hi[:, None])
    mask[:Lv, :Lv] = ok
    if has_text:
        mask[:Lv, Lv:Lv + text_len] = True
        mask[Lv:, :Lv] = True
        mask[Lv:, Lv:Lv + text_len] = True
    return mask


def swa3d_retained_pairs(T, H, W, window, text_len, has_text):
    """Allowed (query, key) pairs of one head."""
    Lv = T * H * W
    n = min(window[0], T) * min(window[1], H) * min(window[2], W)
    total = Lv * (n + (text_len if has_text else 0))
    if has_text:
        total += TEXT_PAD * (Lv + text_len)
    return total
