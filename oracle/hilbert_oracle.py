"""Hilbert-curve token order and block statistics of 2-D local attention
(oracle side).

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

Source: the "Hilbert-guided block-sparse local attention" blog page: image
tokens are reordered along a Hilbert curve, so that 2-D local windows become
contiguous runs of the 1-D sequence; a block-sparse kernel then finds more
empty (skipped) blocks and fewer partial (masked) blocks than with the
row-by-row order.  "Slide attention" is the sliding neighbourhood: every
query token attends to the keys of a window centred on it.

Readings (the page gives no formulas):
  * the grid is n x n tokens, n a power of two; the curve is the standard
    Hilbert curve built by recursive quadrant rotation, starting at (0, 0)
    and ending at (n-1, 0) (x = column, y = row);
  * the slide window is w x w tokens centred on the query and shifted inward
    at the border (as for the token windows of the 3-D comparison);
  * blocks are runs of 128 consecutive tokens of the 1-D order.
"""
import numpy as np


def hilbert_d2xy(n, d):
    """Cell (x, y) at position d along the Hilbert curve of an n x n grid.

    Walks from the finest level up: at each level s the two bits of d select
    a quadrant; the cell found so far is rotated / reflected into the frame
    of that quadrant and offset into it.
    """
    x = y = 0
    t = d
    s = 1
    while s < n:
        rx = (t >> 1) & 1
        ry = (t ^ rx) & 1
        if ry == 0:              # lower quadrants are transposed (and flipped)
            if rx == 1:
                x, y = s - 1 - x, s - 1 - y
            x, y = y, x
        x += s * rx
        y += s * ry
        t >>= 2
        s <<= 1
    return x, y


def hilbert_order(n):
    """Raster index (y * n + x) of the token at each Hilbert position."""
    out = np.empty(n * n, dtype=np.int64)
    for d in range(n * n):
        x, y = hilbert_d2xy(n, d)
        out[d] = y * n + x
    return out


def raster_order(n):
    return np.arange(n * n, dtype=np.int64)


def window_bounds(n, window):
    """[lo, hi) of the centred, border-shifted window along one axis, per coordinate."""
    we = min(window, n)
    c = np.arange(n)
    lo = np.clip(c - we // 2, 0, n - we)
    return lo, lo + we


def slide_mask(n, window, order):
    """Boolean [N, N] mask in the given 1-D order: query i may see key j."""
    lo, hi = window_bounds(n, window)
    ys, xs = order // n, order % n
    okx = (xs[None, :] >= lo[xs][:, None]) & (xs[None, :] < hi[xs][:, None])
    oky = (ys[None, :] >= lo[ys][:, None]) & (ys[None, :] < hi[ys][:, None])
    return okx & oky


def block_classes(n, window, order, block=128):
    """[nb, nb] int8: 0 empty, 1 partial, 2 full (brute force over all pairs)."""
    m = slide_mask(n, window, order)
    nb = (n * n) // block
    cnt = m.reshape(nb, block, nb, block).sum(axis=(1, 3))
    cls = np.where(cnt == 0, 0, np.where(cnt == block * block, 2, 1)).astype(np.int8)
    return cls


def block_rectangles(n, order, block=128):
    """(x0, x1, y0, y1) inclusive bounds of every block, asserting that each
    block is a full rectangle (true for Hilbert blocks of 2 * 4^k tokens and
    for raster blocks that are whole rows or row fragments)."""
    nb = (n * n) // block
    rects = np.empty((nb, 4), dtype=np.int64)
    for b in range(nb):
        ys, xs = order[b * block:(b + 1) * block] // n, order[b * block:(b + 1) * block] % n
        rects[b] = (xs.min(), xs.max(), ys.min(), ys.max())
        assert (xs.max() - xs.min() + 1) * (ys.max() - ys.min() + 1) == block
    return rects


def block_classes_rect(n, window, order, block=128):
    """Same result as block_classes for rectangular blocks, by counting per
    query token the keys of each key rectangle inside its window box."""
    lo, hi = window_bounds(n, window)
    rects = block_rectangles(n, order, block)
    nb = rects.shape[0]
    ys, xs = order // n, order % n
    cls = np.empty((nb, nb), dtype=np.int8)
    for qb in range(nb):
        qx, qy = xs[qb * block:(qb + 1) * block], ys[qb * block:(qb + 1) * block]
        ox = np.minimum(hi[qx][:, None], rects[None, :, 1] + 1) - np.maximum(lo[qx][:, None], rects[None, :, 0])
        oy = np.minimum(hi[qy][:, None], rects[None, :, 3] + 1) - np.maximum(lo[qy][:, None], rects[None, :, 2])
        cnt = (np.clip(ox, 0, None) * np.clip(oy, 0, None)).sum(axis=0)
        cls[qb] = np.where(cnt == 0, 0, np.where(cnt == block * block, 2, 1))
    return cls
