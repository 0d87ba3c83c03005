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


def sta_backward_key_rows(q, k, v, dout, keys_wanted, T, H, W, tile, window, text_len,
                          has_text):
    """dK, dV of the given key rows: every query that attends to one of them
    is found by scanning the allowed-key sets of all query rows."""
    S, d = q.shape
    scale = 1.0 / np.sqrt(d)
    want = {int(j): pos for pos, j in enumerate(keys_wanted)}
    dk = np.zeros((len(keys_wanted), d))
    dv = np.zeros((len(keys_wanted), d))
    # query rows whose allowed set meets the wanted keys (tiles share sets)
    for r in range(S):
        keys = sta_oracle.allowed_keys(r, T, H, W, tile, window, text_len, has_text)
        hit = [j for j in keys_wanted if j in set(keys.tolist())] if len(want) < 8 else \
            np.intersect1d(keys, np.asarray(keys_wanted)).tolist()
        if not hit:
            continue
        (_, p, o, _), = _rows_fwd(q, k, v, [r], T, H, W, tile, window, text_len, has_text)
        dp = v[keys] @ dout[r]
        delta = dout[r] @ o
        ds = p * (dp - delta)
        index = {int(j): c for c, j in enumerate(keys)}
        for j in hit:
            c = index[int(j)]
            dv[want[int(j)]] += p[c] * dout[r]
            dk[want[int(j)]] += ds[c] * q[r] * scale
    return dk, dv
