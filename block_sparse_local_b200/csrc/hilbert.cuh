// hilbert.cuh - Hilbert-curve token order for 2-D local attention and the
// block lists of block-sparse slide attention in a given token order.
//
// "Hilbert-guided block-sparse local attention" (blog page): reordering the
// tokens of an image along a Hilbert curve keeps 2-D neighbourhoods close in
// the 1-D sequence, so a block-sparse kernel meets more empty blocks and fewer
// partial ones than with the row-by-row order.  Slide attention: each query
// token sees the keys of a w x w window centred on it (shifted inward at the
// border).
//
// Curve: n x n grid (n a power of two), position d -> cell (x, y) by walking
// the two-bit digits of d from the finest level up; at each level the cell is
// transposed (and reflected for the last quadrant) into the frame of its
// quadrant, then offset into the quadrant.  Starts at (0, 0), ends at
// (n-1, 0); consecutive positions are 4-neighbours.
#pragma once

#include <cstdint>

namespace sta {

__device__ __forceinline__ void hilbert_cell(int log2n, uint32_t d, int& x, int& y) {
  x = 0;
  y = 0;
  uint32_t t = d;
  for (int lvl = 0; lvl < log2n; ++lvl) {
    const int s = 1 << lvl;
    const int rx = (t >> 1) & 1;
    const int ry = (t ^ rx) & 1;
    if (ry == 0) {
      if (rx == 1) {
        x = s - 1 - x;
        y = s - 1 - y;
      }
      const int tmp = x;
      x = y;
      y = tmp;
    }
    x += s * rx;
    y += s * ry;
    t >>= 2;
  }
}

// Raster index (y * n + x) of the token at position `pos` of the order
// (order 0: raster, 1: Hilbert).
__device__ __forceinline__ int order_to_raster(int order, int log2n, int pos) {
  if (order == 0) return pos;
  int x, y;
  hilbert_cell(log2n, static_cast<uint32_t>(pos), x, y);
  return (y << log2n) + x;
}

// Permutes [slices, n*n, d] rows between raster and Hilbert order
// (to_hilbert: out[pos] = in[raster(pos)], else out[raster(pos)] = in[pos]).
// kVec 16-byte vectors per row; consecutive threads take consecutive vectors.
template <int kVec>
__global__ void __launch_bounds__(256) hilbert_permute_kernel(
    const uint4* __restrict__ in, uint4* __restrict__ out, int log2n, long long total_vec,
    int to_hilbert) {
  const int N = 1 << (2 * log2n);
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total_vec;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long row = i / kVec;
    const int vec = static_cast<int>(i - row * kVec);
    const long long slice = row / N;
    const int pos = static_cast<int>(row - slice * N);
    const int ras = order_to_raster(1, log2n, pos);
    const long long a = (slice * N + pos) * kVec + vec;
    const long long b = (slice * N + ras) * kVec + vec;
    if (to_hilbert)
      out[a] = __ldg(in + b);
    else
      out[b] = __ldg(in + a);
  }
}

// coords[pos] = x | (y << 16) of the token at position pos of the order.
__global__ void __launch_bounds__(256) order_coords_kernel(uint32_t* __restrict__ coords,
                                                           int log2n, int order) {
  const int N = 1 << (2 * log2n);
  const int pos = blockIdx.x * blockDim.x + threadIdx.x;
  if (pos >= N) return;
  const int r = order_to_raster(order, log2n, pos);
  coords[pos] = static_cast<uint32_t>(r & ((1 << log2n) - 1)) |
                (static_cast<uint32_t>(r >> log2n) << 16);
}

// Bounding rectangle (x0, x1, y0, y1), inclusive, of every 128-token block.
// One warp per block.
__global__ void __launch_bounds__(256) block_rect_kernel(const uint32_t* __restrict__ coords,
                                                         int4* __restrict__ rects, int nblocks) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= nblocks) return;
  int x0 = 1 << 30, x1 = -1, y0 = 1 << 30, y1 = -1;
  for (int i = lane; i < 128; i += 32) {
    const uint32_t c = coords[warp * 128 + i];
    const int x = c & 0xffff, y = c >> 16;
    x0 = min(x0, x); x1 = max(x1, x);
    y0 = min(y0, y); y1 = max(y1, y);
  }
  for (int o = 16; o > 0; o >>= 1) {
    x0 = min(x0, __shfl_xor_sync(0xffffffffu, x0, o));
    x1 = max(x1, __shfl_xor_sync(0xffffffffu, x1, o));
    y0 = min(y0, __shfl_xor_sync(0xffffffffu, y0, o));
    y1 = max(y1, __shfl_xor_sync(0xffffffffu, y1, o));
  }
  if (lane == 0) rects[warp] = make_int4(x0, x1, y0, y1);
}

// Window [lo, hi) of coordinate c along an axis of n tokens (w <= n).
__device__ __forceinline__ void slide_bounds(int c, int w, int n, int& lo, int& hi) {
  lo = c - w / 2;
  lo = lo < 0 ? 0 : (lo > n - w ? n - w : lo);
  hi = lo + w;
}

// Key-block lists of 2-D slide attention in a given order.  One CTA of 256
// threads per query group of `qblocks` consecutive 128-token blocks (1 for the
// public per-block lists, 2 for the attention kernel's pairs, which use the
// union).  For every key block the number of allowed (query, key) pairs is
// counted exactly from the block rectangles (every block of the supported
// orders is a full rectangle): class 0 empty, 1 partial, 2 full.  Non-empty
// key blocks are written in ascending order; cls may be null.
__global__ void __launch_bounds__(256) slide_block_list_kernel(
    int* __restrict__ counts, int* __restrict__ ids, int* __restrict__ cls, int max_k,
    const uint32_t* __restrict__ coords, const int4* __restrict__ rects, int nblocks, int n,
    int w, int qblocks) {
  extern __shared__ int sh[];
  int* qlo = sh;                       // [2][256] window x lo, y lo of each query
  int* flag = sh + 2 * 256;            // [nblocks] class of each key block
  __shared__ int warp_sums[8];
  const int grp = blockIdx.x;
  const int nq = 128 * qblocks;
  const int we = w < n ? w : n;
  for (int i = threadIdx.x; i < nq; i += blockDim.x) {
    const uint32_t c = coords[grp * nq + i];
    int lo, hi;
    slide_bounds(static_cast<int>(c & 0xffff), we, n, lo, hi);
    qlo[i] = lo;
    slide_bounds(static_cast<int>(c >> 16), we, n, lo, hi);
    qlo[256 + i] = lo;
  }
  __syncthreads();
  for (int kb = threadIdx.x; kb < nblocks; kb += blockDim.x) {
    const int4 r = rects[kb];
    long long cnt = 0;
    for (int i = 0; i < nq; ++i) {
      const int xl = qlo[i], yl = qlo[256 + i];
      const int ox = min(xl + we, r.y + 1) - max(xl, r.x);
      const int oy = min(yl + we, r.w + 1) - max(yl, r.z);
      if (ox > 0 && oy > 0) cnt += static_cast<long long>(ox) * oy;
    }
    flag[kb] = cnt == 0 ? 0 : (cnt == static_cast<long long>(nq) * 128 ? 2 : 1);
  }
  __syncthreads();
  // ordered compaction: thread t owns key blocks [t*per, (t+1)*per)
  const int per = (nblocks + blockDim.x - 1) / blockDim.x;
  const int b0 = threadIdx.x * per;
  const int b1 = min(b0 + per, nblocks);
  int mine = 0;
  for (int b = b0; b < b1; ++b) mine += flag[b] != 0;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int incl = mine;
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_sums[wid] = incl;
  __syncthreads();
  int before = 0;
  for (int i = 0; i < wid; ++i) before += warp_sums[i];
  int pos = before + incl - mine;
  int* out = ids + static_cast<size_t>(grp) * max_k;
  int* outc = cls ? cls + static_cast<size_t>(grp) * max_k : nullptr;
  for (int b = b0; b < b1; ++b) {
    if (flag[b] != 0 && pos < max_k) {
      out[pos] = b;
      if (outc) outc[pos] = flag[b];
      ++pos;
    }
  }
  int total = 0;
  for (int i = 0; i < 8; ++i) total += warp_sums[i];
  if (threadIdx.x == 0) counts[grp] = total;
  for (int i = total + threadIdx.x; i < max_k; i += blockDim.x) {
    out[i] = -1;
    if (outc) outc[i] = 0;
  }
}

}  // namespace sta
