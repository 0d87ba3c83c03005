// tile_lists.cuh - per-query-tile KV tile lists (integer, bit-exact).
//
// STA README, Usage: "window_size in tiles", one (window_t, window_h,
// window_w) per entry of the list; a (3,3,3) window lets a query see
// (3x6, 3x8, 3x8) tokens, i.e. every query tile sees a full box of tiles.
// The box is centred on the query tile (start c - floor(w/2)) and shifted
// inward at the border; a window longer than an axis covers the axis.
//
// Row r < NV of window class c lists the key tiles of the box in ascending
// tile id ((t*NH + h)*NW + w, so the t-h-w loop nest below is ascending),
// then the text sentinel NV when the text block holds valid keys.  Row NV
// (present when has_text) is the text query block: every video tile, then
// the sentinel.  Unused slots up to max_k are -1.
#pragma once

#include "device_ptx.cuh"

namespace sta {

constexpr int kMaxWindowClasses = 256;

// Windows passed by value (kernel parameter space), [class][3] in tiles.
struct ListWindows {
  int w[3 * kMaxWindowClasses];
};

struct ListGeom {
  int NT, NH, NW;
  int NV;
  int NQ;          // rows per window class (NV, or NV + 1 with text)
  int max_k;
  int text_block;  // 1 when the text block has valid keys
  int token_mode;  // windows counted in tokens (3-D sliding window), not tiles
  int ct, ch, cw;  // tile size (token mode)
};

__device__ __forceinline__ void window_range(int c, int w, int n, int& s,
                                             int& e) {
  e = w < n ? w : n;
  s = c - e / 2;
  if (s < 0) s = 0;
  if (s > n - e) s = n - e;
}

// Token-window mode: the key tiles that hold any key of the windows of the
// tokens of query tile c along one axis.  Token windows are centred on the
// token and shifted inward at the border; their starts grow with the token,
// so the first and last token of the tile bound the union.
__device__ __forceinline__ void token_tile_range(int c, int w, int cs, int n, int& s,
                                                 int& e) {
  const int X = n * cs;
  const int we = w < X ? w : X;
  int lo = c * cs - we / 2;
  lo = lo < 0 ? 0 : (lo > X - we ? X - we : lo);
  int hi = c * cs + cs - 1 - we / 2;
  hi = hi < 0 ? 0 : (hi > X - we ? X - we : hi);
  s = lo / cs;
  e = (hi + we - 1) / cs - s + 1;
}

// One thread per (class, row).
__global__ void __launch_bounds__(128) kv_tile_list_kernel(
    int* __restrict__ counts, int* __restrict__ ids, const ListWindows windows,
    int nclass, ListGeom g) {
  const int gid = blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= nclass * g.NQ) return;
  const int cls = gid / g.NQ;
  const int row = gid - cls * g.NQ;
  int* out = ids + static_cast<size_t>(gid) * g.max_k;
  int n = 0;
  if (row < g.NV) {
    const int qw = row % g.NW;
    const int qh = (row / g.NW) % g.NH;
    const int qt = row / (g.NW * g.NH);
    int st, et, sh, eh, sw, ew;
    if (g.token_mode) {
      token_tile_range(qt, windows.w[cls * 3 + 0], g.ct, g.NT, st, et);
      token_tile_range(qh, windows.w[cls * 3 + 1], g.ch, g.NH, sh, eh);
      token_tile_range(qw, windows.w[cls * 3 + 2], g.cw, g.NW, sw, ew);
    } else {
      window_range(qt, windows.w[cls * 3 + 0], g.NT, st, et);
      window_range(qh, windows.w[cls * 3 + 1], g.NH, sh, eh);
      window_range(qw, windows.w[cls * 3 + 2], g.NW, sw, ew);
    }
    for (int t = st; t < st + et; ++t)
      for (int h = sh; h < sh + eh; ++h)
        for (int w = sw; w < sw + ew; ++w)
          if (dbg_ok(n < g.max_k)) out[n++] = (t * g.NH + h) * g.NW + w;
  } else {
    for (int t = 0; t < g.NV; ++t)
      if (dbg_ok(n < g.max_k)) out[n++] = t;
  }
  if (g.text_block && dbg_ok(n < g.max_k)) out[n++] = g.NV;
  counts[gid] = n;
  for (int i = n; i < g.max_k; ++i) out[i] = -1;
}

}  // namespace sta
