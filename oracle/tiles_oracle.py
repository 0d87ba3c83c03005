"""Per-query-tile KV tile lists, by brute force (oracle side).

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

README "Sliding Tile Atteniton Kernel", Usage (the window is counted in
tiles) and "Why is STA Fast?" (STA has no partially masked blocks): a query
tile attends to whole key tiles, so the work of one query tile is a list of
key tiles.

Encoding (the library's bit-exact contract):
  * tiles are numbered in tile-major raster order,
    id = (tile_t * NH + tile_h) * NW + tile_w, NV = NT*NH*NW tiles;
  * row r < NV lists, in ascending order, every key tile k whose box test
    passes on all three axes, then the sentinel NV (the text block) when
    has_text and text_len > 0;
  * when has_text, row NV is the text query block: every video tile
    0..NV-1, then the sentinel NV when text_len > 0;
  * counts[h][r] is the list length, ids[h][r][count:max_k] are -1.
"""
import numpy as np

from .geometry import tile_grid, window_start


def kv_tile_lists(T, H, W, tile, windows, text_len, has_text, max_k=None):
    """Return (counts [heads, NQ] int32, ids [heads, NQ, max_k] int32).

    Brute force: for every (query tile, key tile) pair, test the window box
    predicate on each axis.
    """
    N = tile_grid(T, H, W, tile)
    NV = N[0] * N[1] * N[2]
    NQ = NV + (1 if has_text else 0)
    heads = len(windows)
    text_block = has_text and text_len > 0
    lists = []
    for h in range(heads):
        per_head = []
        for q in range(NV):
            qc = (q // (N[1] * N[2]), (q // N[2]) % N[1], q % N[2])
            row = []
            for kt in range(NV):
                kc = (kt // (N[1] * N[2]), (kt // N[2]) % N[1], kt % N[2])
                inside = True
                for a in range(3):
                    s, e = window_start(qc[a], windows[h][a], N[a])
                    if not (s <= kc[a] < s + e):
                        inside = False
                        break
                if inside:
                    row.append(kt)
            if text_block:
                row.append(NV)
            per_head.append(row)
        if has_text:
            per_head.append(list(range(NV)) + ([NV] if text_block else []))
        lists.append(per_head)
    need = max(len(r) for ph in lists for r in ph)
    if max_k is None:
        max_k = need
    if max_k < need:
        raise ValueError("max_k too small")
    counts = np.zeros((heads, NQ), dtype=np.int32)
    ids = np.full((heads, NQ, max_k), -1, dtype=np.int32)
    for h in range(heads):
        for r, row in enumerate(lists[h]):
            counts[h, r] = len(row)
            ids[h, r, :len(row)] = row
    return counts, ids
