"""Tile geometry of STA, written out from its definition (oracle side).

README "Sliding Tile Atteniton Kernel", section Usage:
  * the video is a (T, H, W) token grid, flattened in raster order;
  * tiles are (6, 8, 8) blocks of tokens (t, h, w);
  * the window is given in tiles: window (3,3,3) lets a query attend to
    (3x6, 3x8, 3x8) = (18, 24, 24) tokens, i.e. a window counts whole tiles
    and every query sees a full window;
  * 256 text tokens (with padding) follow the video tokens;
    ``text_length`` ranges over 0..256.

Readings taken where the page is silent:
  * the window is centred on the query tile, start = c - floor(w/2), and
    shifted inward at the grid border so that it always spans w tiles
    (pinned for odd windows by the hand-derived fixtures; for an even window
    shorter than the grid the choice of the extra tile on the low side is
    parity unpinned: no page example fixes it);
  * a window longer than the grid axis is clipped to the whole axis;
  * with has_text=False there are no text rows at all.
"""

TEXT_PAD = 256  # README Usage: the text block is padded to 256 tokens


def tile_grid(T, H, W, tile):
    ct, ch, cw = tile
    if T % ct or H % ch or W % cw:
        raise ValueError("video grid must be a whole number of tiles")
    return (T // ct, H // ch, W // cw)


def window_start(c, w, n):
    """Start tile and extent of the window along one axis.

    c: query tile coordinate on this axis, w: window length in tiles,
    n: number of tiles on this axis.  Returns (s, we) with the window being
    tiles s .. s+we-1.
    """
    we = min(w, n)
    s = c - we // 2
    if s < 0:
        s = 0
    if s > n - we:
        s = n - we
    return s, we


def seq_len(T, H, W, has_text):
    return T * H * W + (TEXT_PAD if has_text else 0)
