// reorder.cuh - raster <-> tile token permutation (bit-exact row copies).
//
// STA README, Usage: tiles are (6, 8, 8) blocks of tokens.  For the
// tile-by-tile blocks of the attention map to be dense ("Why is STA Fast?")
// the tokens of one tile must be contiguous rows.  Video row
// r = (t*H + h)*W + w lives at tile-ordered row tile_id*V + in_tile with
//   tile_id = ((t/ct)*NH + h/ch)*NW + w/cw,
//   in_tile = ((t%ct)*ch + h%ch)*cw + w%cw,   V = ct*ch*cw.
// Text rows (after the video) keep their position.
//
// One CTA moves one tile of one (batch, head) slice: tile coordinates are
// computed once per CTA, the in-tile coordinates with multiply-shift
// division.  Every row is d*2 bytes moved as 16-byte vectors; consecutive
// threads take consecutive vectors, so each warp reads and writes whole
// contiguous rows (runs of cw rows are contiguous on the raster side).
#pragma once

#include "device_ptx.cuh"

#include <cstdint>

namespace sta {

// Division by a runtime constant 1 <= d < 2^31 for 0 <= x < 2^31 with one
// multiply-high, an add and a shift (Granlund & Montgomery, "Division by
// invariant integers using multiplication", PLDI 1994, round-up variant).
struct FastDiv {
  uint32_t div, mul, shr;
};

inline FastDiv make_fastdiv(uint32_t d) {
  FastDiv f;
  f.div = d;
  uint32_t l = 0;
  while ((1ull << l) < d) ++l;
  f.shr = l;
  f.mul = static_cast<uint32_t>(((1ull << 32) * ((1ull << l) - d)) / d + 1ull);
  return f;
}

__device__ __forceinline__ uint32_t fdiv(uint32_t x, const FastDiv& f) {
  uint32_t hi = __umulhi(x, f.mul);
  return (hi + x) >> f.shr;
}

struct ReorderGeom {
  int T, H, W;
  int ct, ch, cw;
  int NH, NW;
  int V;                 // tile volume
  int S;                 // rows per slice
  int Lv;                // video rows per slice
  int num_tiles;         // NV
  FastDiv div_cw, div_chcw;
};

// Grid: x = tile id (0..NV-1; NV = the text block when present), y = slice.
// kVec: 16-byte vectors per row (d*2/16).  to_tile=1: raster -> tile order.
template <int kVec>
__global__ void __launch_bounds__(256) tile_permute_kernel(
    const uint4* __restrict__ in, uint4* __restrict__ out, ReorderGeom g,
    int to_tile) {
  const int tile = blockIdx.x;
  const size_t slice_base = static_cast<size_t>(blockIdx.y) * g.S;
  if (tile >= g.num_tiles) {
    // text block: identity copy of rows Lv .. S-1
    const int rows = g.S - g.Lv;
    const int n = rows * kVec;
    const size_t base = (slice_base + g.Lv) * kVec;
    const size_t total = static_cast<size_t>(gridDim.y) * g.S * kVec;
    for (int i = threadIdx.x; i < n; i += blockDim.x)
      if (dbg_ok(base + i < total)) out[base + i] = in[base + i];
    return;
  }
  const int tw = tile % g.NW;
  const int th = (tile / g.NW) % g.NH;
  const int tt = tile / (g.NW * g.NH);
  const int t0 = tt * g.ct, h0 = th * g.ch, w0 = tw * g.cw;
  const size_t tile_row0 = slice_base + static_cast<size_t>(tile) * g.V;
  const int n = g.V * kVec;
  constexpr int kUnroll = 4;
  for (int base = threadIdx.x; base < n; base += blockDim.x * kUnroll) {
    uint4 v[kUnroll];
    size_t dst[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int i = base + u * blockDim.x;
      if (i < n) {
        const uint32_t row = static_cast<uint32_t>(i) / kVec;
        const uint32_t vec = static_cast<uint32_t>(i) % kVec;
        const uint32_t q1 = fdiv(row, g.div_cw);      // row / cw
        const uint32_t iw = row - q1 * g.cw;
        const uint32_t it = fdiv(row, g.div_chcw);    // row / (ch*cw)
        const uint32_t ih = q1 - it * g.ch;
        const size_t raster = slice_base +
            (static_cast<size_t>(t0 + it) * g.H + (h0 + ih)) * g.W + (w0 + iw);
        const size_t tiled = tile_row0 + row;
        const size_t src = (to_tile ? raster : tiled) * kVec + vec;
        dst[u] = (to_tile ? tiled : raster) * kVec + vec;
        const size_t total = static_cast<size_t>(gridDim.y) * g.S * kVec;
        v[u] = dbg_ok(src < total) ? __ldg(in + src) : make_uint4(0u, 0u, 0u, 0u);
        if (!dbg_ok(dst[u] < total)) dst[u] = total;   // marks the store as skipped
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int i = base + u * blockDim.x;
      if (i < n && (!STA_DEBUG || dst[u] < static_cast<size_t>(gridDim.y) * g.S * kVec))
        out[dst[u]] = v[u];
    }
  }
}

}  // namespace sta
