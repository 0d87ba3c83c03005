"""Raster <-> tile token permutation (oracle side).

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

README "Sliding Tile Atteniton Kernel", Usage: tiles are (6, 8, 8) blocks of
tokens.  A tile's tokens have to be contiguous rows of q, k, v for the
tile-by-tile blocks of the attention map to be dense ("Why is STA Fast?").
Reading (the page does not fix the order): tiles in tile-major raster order,
tokens inside a tile in raster order, text rows left in place.

Index formula: video token (t, h, w) at raster row r = (t*H + h)*W + w moves
to row p = tile_id * V + in_tile with
  tile_id = ((t // ct) * NH + h // ch) * NW + w // cw,
  in_tile = ((t % ct) * ch + h % ch) * cw + w % cw,   V = ct*ch*cw.
"""
import numpy as np

from .geometry import tile_grid


def tile_position_of_raster(T, H, W, tile):
    """p[r]: tile-ordered row of raster video row r (the formula above)."""
    ct, ch, cw = tile
    NT, NH, NW = tile_grid(T, H, W, tile)
    r = np.arange(T * H * W, dtype=np.int64)
    t, h, w = r // (H * W), (r // W) % H, r % W
    tile_id = ((t // ct) * NH + h // ch) * NW + w // cw
    in_tile = ((t % ct) * ch + h % ch) * cw + w % cw
    return tile_id * (ct * ch * cw) + in_tile


def reorder(x, T, H, W, tile, has_text):
    """x: [..., S, d] raster order -> tile order (text rows unchanged)."""
    Lv = T * H * W
    p = tile_position_of_raster(T, H, W, tile)
    out = x.copy()
    out[..., p, :] = x[..., :Lv, :]
    return out


def unreorder(x, T, H, W, tile, has_text):
    """Inverse of reorder."""
    Lv = T * H * W
    p = tile_position_of_raster(T, H, W, tile)
    out = x.copy()
    out[..., :Lv, :] = x[..., p, :]
    return out
