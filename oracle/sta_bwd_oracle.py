"""Backward pass of STA in float64 (oracle side).

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

The STA pages describe only the forward computation; the backward pass is the
gradient of that same function (masked softmax attention, mask as in
oracle/sta_oracle.py), written out step by step:
  S = q k^T / sqrt(d) on allowed pairs,  P = softmax_rows(S),  O = P v
  dV = P^T dO
  dP = dO v^T
  D_i = sum_j P_ij dP_ij  ( = sum_c dO_ic O_ic )
  dS = P * (dP - D)
  dQ = dS k / sqrt(d),   dK = dS^T q / sqrt(d)
Padded text keys (u >= text_len) are attended by no query, so their dK and
dV rows are zero.
"""
import numpy as np

from . import sta_oracle


def sta_backward_dense(q, k, v, dout, T, H, W, tile, window, text_len, has_text):
    """One (batch, head): q, k, v, dout float64 [S, d] raster order.

    Returns (dq, dk, dv, out, lse)."""
    d = q.shape[1]
    scale = 1.0 / np.sqrt(d)
    mask = sta_oracle.sta_mask(T, H, W, tile, window, text_len, has_text)
    out, lse, p = sta_oracle.masked_softmax_attention(q, k, v, mask, scale)
    dv = p.T @ dout
    dp = dout @ v.T
    delta = (dout * out).sum(axis=1, keepdims=True)
    ds = p * (dp - delta)
    dq = (ds @ k) * scale
    dk = (ds.T @ q) * scale
    return dq, dk, dv, out, lse


def _rows_fwd(q, k, v, rows, T, H, W, tile, window, text_len, has_text):
    """Forward quantities of the given query rows: list of (keys, P, O, lse)."""
    d = q.shape[1]
    scale = 1.0 / np.sqrt(d)
    res = []
    for r in rows:
        keys = sta_oracle.allowed_keys(int(r), T, H, W, tile, window, text_len, has_text)
        s = (k[keys] @ q[r]) * scale
        m = s.max()
        e = np.exp(s - m)
        l = e.sum()
        p = e / l
        res.append((keys, p, p @ v[keys], m + np.log(l)))
    return res


def sta_backward_query_rows(q, k, v, dout, rows, T, H, W, tile, window, text_len, has_text):
    """dQ of the given query rows (one (batch, head), raster order)."""
    d = q.shape[1]
    scale = 1.0 / np.sqrt(d)
    dq = np.empty((len(rows), d))
    for pos, (r, (keys, p, o, _)) in enumerate(
            zip(rows, _rows_fwd(q, k, v, rows, T, H, W, tile, window, text_len, has_text))):
        dp = v[keys] @ dout[r]
        delta = dout[r] @ o
        ds = p * (dp - delta)
        dq[pos] = (ds @ k[keys]) * scale
    return dq


def _query_groups(T, H, W, tile, has_text):
    """Query rows grouped by the key set they share: the raster rows of each
    video query tile, then (with text) the 256 text rows."""
    N = sta_oracle.tile_grid(T, H, W, tile)
    groups = []
    for t in range(N[0]):
        for h in range(N[1]):
            for w in range(N[2]):
                groups.append(np.sort(sta_oracle._box_rows(T, H, W, tile, (t, h, w),
                                                           (1, 1, 1))))
    if has_text:
        Lv = T * H * W
        groups.append(np.arange(Lv, Lv + sta_oracle.TEXT_PAD))
    return groups


def sta_backward_key_rows(q, k, v, dout, keys_wanted, T, H, W, tile, window, text_len,
                          has_text):
    """dK, dV of the given key rows (one (batch, head), raster order).

    Every query row whose allowed set holds a wanted key contributes; rows of
    one query tile (and the text rows) share their allowed set, so each such
    group is one gather: S, P, O, dP and dS of the group's rows over its
    allowed keys, then the wanted keys' columns of P^T dO and dS^T q."""
    S, d = q.shape
    scale = 1.0 / np.sqrt(d)
    wanted = np.asarray(keys_wanted, dtype=np.int64)
    dk = np.zeros((len(wanted), d))
    dv = np.zeros((len(wanted), d))
    for rows in _query_groups(T, H, W, tile, has_text):
        keys = sta_oracle.allowed_keys(int(rows[0]), T, H, W, tile, window, text_len, has_text)
        hit = np.isin(wanted, keys)
        if not hit.any():
            continue
        s = (q[rows] @ k[keys].T) * scale
        p = np.exp(s - s.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        o = p @ v[keys]
        dp = dout[rows] @ v[keys].T
        delta = (dout[rows] * o).sum(axis=1, keepdims=True)
        ds = p * (dp - delta)
        cols = np.searchsorted(keys, wanted[hit])
        dv[hit] += p[:, cols].T @ dout[rows]
        dk[hit] += (ds[:, cols].T @ q[rows]) * scale
    return dk, dv
