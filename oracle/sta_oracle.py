"""STA forward in float64: the plain definition, in raster token order.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

What STA computes (README "Sliding Tile Atteniton Kernel", Usage and
"Why is STA Fast?"): exact softmax attention softmax(q k^T / sqrt(d)) v in
which a query token may only see key tokens whose tile lies inside the window
of tiles around the query's own tile; the attention map is made of whole
tile-by-tile blocks that are either fully dense or fully empty.

Mask rule, for query token i and key token j (raster order, L_v video tokens
followed by the padded text block of 256 rows):
  1. both video: allowed iff, on every axis a, the key's tile coordinate lies
     in [s_a, s_a + w'_a) where (s_a, w'_a) = window_start(query tile c_a, ...);
  2. video query, text key L_v+u: allowed iff has_text and u < text_len;
  3. text query (i >= L_v): allowed iff j is a video key, or a text key with
     u < text_len.  (Padded text query rows u >= text_len follow the same
     rule as valid text rows.)
Rules 2 and 3 are the reading taken for the optional text tokens that the
README's Usage section appends after the video; the page gives no formula for
them.

Two independent forms are provided and cross-checked by the tests:
  * form A: an explicit S x S boolean mask and a masked softmax (tiny only);
  * form B: per query tile, gather the allowed key rows and do one float64
    matmul (scales to sampled rows of the full workloads).
Both return the output and the natural-log log-sum-exp of each row.
"""
import numpy as np

from .geometry import TEXT_PAD, tile_grid, window_start, seq_len


# ----------------------------------------------------------------------------
# form A: explicit dense mask
# ----------------------------------------------------------------------------
def sta_mask(T, H, W, tile, window, text_len, has_text):
    """S x S boolean mask (True = attended), rules 1-3 above."""
    ct, ch, cw = tile
    N = tile_grid(T, H, W, tile)
    Lv = T * H * W
    S = seq_len(T, H, W, has_text)
    r = np.arange(Lv)
    coord = (r // (H * W), (r // W) % H, r % W)
    tcoord = (coord[0] // ct, coord[1] // ch, coord[2] // cw)
    vv = np.ones((Lv, Lv), dtype=bool)
    for a in range(3):
        lo = np.empty(Lv, dtype=np.int64)
        ext = np.empty(Lv, dtype=np.int64)
        for idx, c in enumerate(tcoord[a]):
            lo[idx], ext[idx] = window_start(int(c), window[a], N[a])
        kc = tcoord[a][None, :]
        vv &= (kc >= lo[:, None]) & (kc < (lo + ext)[:, None])
    mask = np.zeros((S, S), dtype=bool)
    mask[:Lv, :Lv] = vv
    if has_text:
        mask[:Lv, Lv:Lv + text_len] = True
        mask[Lv:, :Lv] = True
        mask[Lv:, Lv:Lv + text_len] = True
    return mask


def masked_softmax_attention(q, k, v, mask, scale):
    """out_i = sum_j softmax_j(scale q_i.k_j | mask) v_j, float64; also LSE."""
    s = (q @ k.T) * scale
    s = np.where(mask, s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    p = np.where(mask, np.exp(s - m), 0.0)
    l = p.sum(axis=1, keepdims=True)
    out = (p @ v) / l
    lse = (m + np.log(l))[:, 0]
    return out, lse, p / l


def sta_forward_dense(q, k, v, T, H, W, tile, window, text_len, has_text):
    """Form A for one (batch, head): q, k, v float64 [S, d] in raster order."""
    d = q.shape[1]
    mask = sta_mask(T, H, W, tile, window, text_len, has_text)
    out, lse, _ = masked_softmax_attention(q, k, v, mask, 1.0 / np.sqrt(d))
    return out, lse


# ----------------------------------------------------------------------------
# form B: gather the allowed keys per query tile
# ----------------------------------------------------------------------------
def _box_rows(T, H, W, tile, starts, exts):
    """Raster indices of the tokens inside a box of tiles."""
    ct, ch, cw = tile
    tt = np.arange(starts[0] * ct, (starts[0] + exts[0]) * ct)
    hh = np.arange(starts[1] * ch, (starts[1] + exts[1]) * ch)
    ww = np.arange(starts[2] * cw, (starts[2] + exts[2]) * cw)
    return ((tt[:, None, None] * H + hh[None, :, None]) * W
            + ww[None, None, :]).reshape(-1)


def allowed_keys(qrow, T, H, W, tile, window, text_len, has_text):
    """Sorted raster indices of the keys query ``qrow`` may attend to."""
    Lv = T * H * W
    if qrow >= Lv:  # rule 3: text query
        keys = np.arange(Lv + text_len)
        return keys
    ct, ch, cw = tile
    N = tile_grid(T, H, W, tile)
    t, h, w = qrow // (H * W), (qrow // W) % H, qrow % W
    c = (t // ct, h // ch, w // cw)
    se = [window_start(c[a], window[a], N[a]) for a in range(3)]
    keys = np.sort(_box_rows(T, H, W, tile, [s for s, _ in se], [e for _, e in se]))
    if has_text and text_len > 0:  # rule 2
        keys = np.concatenate([keys, Lv + np.arange(text_len)])
    return keys


def _query_tile_of(row, T, H, W, tile):
    Lv = T * H * W
    if row >= Lv:
        return -1
    ct, ch, cw = tile
    N = tile_grid(T, H, W, tile)
    t, h, w = row // (H * W), (row // W) % H, row % W
    return ((t // ct) * N[1] + h // ch) * N[2] + w // cw


def sta_forward_rows(q, k, v, T, H, W, tile, window, text_len, has_text,
                     rows=None):
    """Form B for one (batch, head).

    q, k, v: float64 [S, d] raster order.  ``rows``: raster query rows to
    compute (default: all).  Returns (out [len(rows), d], lse [len(rows)]).
    Rows are grouped by query tile so each group is one gather + one matmul.
    """
    S, d = q.shape
    if S != seq_len(T, H, W, has_text):
        raise ValueError("sequence length does not match the grid")
    scale = 1.0 / np.sqrt(d)
    rows = np.arange(S) if rows is None else np.asarray(rows, dtype=np.int64)
    out = np.empty((len(rows), d), dtype=np.float64)
    lse = np.empty(len(rows), dtype=np.float64)
    groups = {}
    for pos, r in enumerate(rows):
        groups.setdefault(_query_tile_of(int(r), T, H, W, tile), []).append(pos)
    for _, poss in groups.items():
        poss = np.asarray(poss)
        keys = allowed_keys(int(rows[poss[0]]), T, H, W, tile, window,
                            text_len, has_text)
        s = (q[rows[poss]] @ k[keys].T) * scale
        m = s.max(axis=1, keepdims=True)
        p = np.exp(s - m)
        l = p.sum(axis=1, keepdims=True)
        out[poss] = (p @ v[keys]) / l
        lse[poss] = (m + np.log(l))[:, 0]
    return out, lse


def sta_forward_batched(q, k, v, T, H, W, tile, windows, text_len, has_text,
                        rows=None, pairs=None):
    """Form B over [B, heads, S, d] float64 inputs with one window per head.

    ``windows``: heads x 3 window sizes in tiles (README Usage gives the
    window as a list of (window_t, window_h, window_w); read here as one
    entry per head).  ``pairs``: iterable of (b, h) to compute (default all).
    Returns dict {(b, h): (out, lse)}.
    """
    Bn, nh = q.shape[0], q.shape[1]
    if pairs is None:
        pairs = [(b, h) for b in range(Bn) for h in range(nh)]
    res = {}
    for b, h in pairs:
        res[(b, h)] = sta_forward_rows(q[b, h], k[b, h], v[b, h], T, H, W, tile,
                                       tuple(windows[h]), text_len, has_text,
                                       rows)
    return res


def retained_pairs(T, H, W, tile, window, text_len, has_text):
    """Number of allowed (query, key) pairs of one head, by counting keys."""
    S = seq_len(T, H, W, has_text)
    Lv = T * H * W
    N = tile_grid(T, H, W, tile)
    ct, ch, cw = tile
    V = ct * ch * cw
    total = 0
    for tq in range(N[0] * N[1] * N[2]):
        c = (tq // (N[1] * N[2]), (tq // N[2]) % N[1], tq % N[2])
        n = 1
        for a in range(3):
            n *= window_start(c[a], window[a], N[a])[1]
        total += V * (n * V + (text_len if has_text else 0))
    if has_text:
        total += (S - Lv) * (Lv + text_len)
    return total
