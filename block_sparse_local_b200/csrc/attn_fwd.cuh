// attn_fwd.cuh - fused block-sparse attention forward for sm_100a.
//
// Computes, for every 128-row query block, O = softmax(Q K^T / sqrt(d)) V over
// a list of 128-key blocks, with tensor cores (tcgen05, accumulators in TMEM)
// and an online softmax in fp32.  Two modes share the pipeline:
//
//  * Mode::kSta - Sliding Tile Attention (STA README, "Usage" and "Why is STA
//    Fast?"): the key blocks of a query tile are the whole key tiles of its
//    window, plus the padded text block.  Video tiles are always dense; only
//    the text block, whose last columns may be padding (text_length < 256),
//    is masked.
//  * Mode::kSwa - token-level causal sliding-window attention with GQA (the
//    mixed-block baseline of "Why is STA Fast?"; window over previous
//    positions as on the sliding-window search-result page).  Blocks cut by
//    the band edges are masked per element.
//
// CTA = 2 + 8 * kSplit warps (18 with kSplit = 2), one work item = up to
// two 128-row query blocks ("slots") that read the same key blocks:
//   warp 0      TMA producer, one lane per operand panel: Q once, then K
//               and V blocks into K / V rings of shared-memory stages
//               (128-byte swizzle).
//   warp 1      MMA issuer (the whole warp waits, one elected lane issues)
//               and TMEM owner: S_i = Q_i K^T (SS, M=128 N=128 K=d),
//               O_i += P_i V (TS: P from TMEM, V from shared memory, N=d),
//               ping-ponging the two slots so the tensor pipe works on one
//               slot while the other slot's softmax runs.
//   warps 2..   softmax, 8 warps per slot, two per TMEM lane quarter, each
//               warp on 16 of the quarter's 32 query rows (TMEM lanes) with
//               two threads per row (lanes t and t + 16), each thread with 64
//               of the row's 128 scores, so the row's max and sum are one
//               warp shuffle away; exponentials two at a time with packed
//               f32x2 arithmetic (a
//               share of them on the FMA pipe) against the running max, the
//               block max taken in the same loop; they update the running
//               max / sum, write bf16 P over the first half of their own
//               score columns, rescale their O columns when the max grew by
//               more than 2^8, and finally normalise O and store it.
// TMEM (512 columns): S0 [0,128), S1 [128,256), O0 [256,256+d),
// O1 [256+d, 256+2d); P_i aliases half of S_i.  The MMA that overwrites S_i
// with the next scores is issued after the P_i.V MMA that reads P_i;
// tcgen05 MMAs of one thread execute in issue order.
#pragma once

#include <type_traits>

#include "device_ptx.cuh"

namespace sta {

constexpr int kBM = 128;        // query rows per block (MMA M)
constexpr int kBN = 128;        // keys per block
// Threads that share one query row's softmax (each takes 128 / kSplit score
// columns of the row, two lanes of one warp); the two slots' softmax use
// 8 * kSplit warps.
constexpr int kSplit = 2;

constexpr int kFwdThreads = 64 + 256 * kSplit;
constexpr int kWarpTma = 0;
constexpr int kWarpMma = 1;
constexpr int kWarpSoftmax0 = 2;

enum class Mode { kSta = 0, kSwa = 1, kSwa3d = 2, kSlide2d = 3 };

struct WorkItem {
  int q0;       // first row (in the [B*heads*S, d] view) of query block 0
  int q1;       // same for block 1, or -1
  int kv_base;  // first row of the key/value slice
  int list;     // kSta: tile-list row; kSwa: query block index
};

// Geometry of raster-ordered q, k, v, out (sta_forward_raster): the kernel
// reads each 128-row block of a tile as a box of the (T, H, W) grid and
// writes each output row to its raster position, so no separate permutation
// pass is needed.
struct RasterGeom {
  int S;            // rows per (batch, head) slice
  int T;            // video grid along t
  int ct, ch, cw;   // tile
  int H, W;         // video grid (T is implied)
  int NH, NW;       // tile grid
};

struct FwdParams {
  const WorkItem* items;
  const int* item_off;  // CTA pairs: items of cluster c are [item_off[c], item_off[c + 1])
  const int* counts;
  const int* ids;
  int max_k;
  int tile_blocks;    // tile volume / 128
  int V;              // tile volume
  int L_v;            // video rows of a slice
  int text_len;       // valid text keys
  int text_blocks;    // key blocks of the text block holding valid keys
  int text_sentinel;  // lists end with the text block
  int window;         // kSwa: tokens
  int win3[3];        // kSwa3d: (Wt, Wh, Ww) token window
  const uint32_t* coords;  // kSlide2d: x | y << 16 of every position of the order
  int grid_n;         // kSlide2d: n of the n x n grid
  int win2;           // kSlide2d: w of the w x w window
  int khalf_t;        // CTA pairs, raster order: key halves split along t (1) or h (0)
  int kbox_t, kbox_h; // CTA pairs, raster order: the 128-row block's box along t, h
  float scale_log2;   // log2(e) / sqrt(d)
  __nv_bfloat16* out;
  float* lse;
  RasterGeom rg;      // used when the kernel runs on raster-ordered tensors
  // extents for the bounds checks of the debug build
  int dbg_rows_q;     // rows of q and out in the [rows, d] view
  int dbg_rows_kv;    // rows of k and v
  int dbg_lists;      // rows of the key-block lists (kSta, kSwa3d, kSlide2d)
};

// Debug build: the work item and its key-block list are inside the arrays
// they index (checked once per CTA before anything is loaded).
template <Mode M>
__device__ __forceinline__ bool item_in_bounds(const FwdParams& p, const WorkItem& it) {
  bool ok = it.q0 >= 0 && it.q0 + kBM <= p.dbg_rows_q;
  ok = ok && (it.q1 < 0 || it.q1 + kBM <= p.dbg_rows_q);
  ok = ok && it.kv_base >= 0 && it.kv_base < p.dbg_rows_kv;
  if constexpr (M != Mode::kSwa) {
    ok = ok && it.list >= 0 && it.list < p.dbg_lists;
    if (ok) {
      const int cnt = p.counts[it.list];
      ok = cnt >= 0 && cnt <= p.max_k;
    }
  }
  return ok;
}

template <int D>
struct FwdCfg {
  static constexpr int kPanels = D / 64;          // 128-byte swizzle panels
  static constexpr int kPanelBytes = 128 * 128;   // 128 rows x 128 bytes
  static constexpr int kBlockBytes = kBM * D * 2;
  static constexpr int kKStages = D == 128 ? 2 : 4;
  static constexpr int kVStages = D == 128 ? 2 : 4;
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + 2 * kBlockBytes;
  static constexpr int kVOff = kKOff + kKStages * kBlockBytes;
  static constexpr int kBarOff = kVOff + kVStages * kBlockBytes;
  static constexpr int kSmemBytes = kBarOff + 512 + 1024;  // + 1024-byte align
  static constexpr uint32_t kTmemCols = 512;
  // Score buffers of 128 columns: one per slot at d = 128 (S0, S1, then
  // O0, O1 fill the 512 columns); at d = 64 the two 64-column O's leave room
  // for a pool of three, so a slot's next Q K^T can run before its P V.
  static constexpr int kSBuf = D == 64 ? 3 : 2;
  static constexpr uint32_t kOCol = kSBuf * 128;
};

// Key-block sequence of one work item, identical for all roles.
struct KvSeq {
  int n;            // number of key blocks
  int nvid;         // kSta: video blocks before the text blocks
  const int* ids;   // kSta: tile ids of the list
  int kv_base;
  int qb;           // kSwa: query block
};

template <Mode M>
__device__ __forceinline__ KvSeq make_seq(const FwdParams& p, const WorkItem& it) {
  KvSeq s;
  s.kv_base = it.kv_base;
  if constexpr (M != Mode::kSwa) {
    const int cnt = p.counts[it.list];
    s.ids = p.ids + static_cast<size_t>(it.list) * p.max_k;
    s.nvid = (cnt - p.text_sentinel) * p.tile_blocks;
    s.n = s.nvid + (p.text_sentinel ? p.text_blocks : 0);
    s.qb = 0;
  } else {
    s.qb = it.list;
    int lo = s.qb * kBN - p.window + 1;     // smallest key of the band
    int kb_lo = lo <= 0 ? 0 : lo / kBN;
    s.n = s.qb - kb_lo + 1;                 // diagonal block first
    s.nvid = s.n;
    s.ids = nullptr;
  }
  return s;
}

template <Mode M>
__device__ __forceinline__ int seq_row(const FwdParams& p, const KvSeq& s, int j) {
  if constexpr (M != Mode::kSwa) {
    if (j < s.nvid) {
      const int t = j / p.tile_blocks;
      return s.kv_base + s.ids[t] * p.V + (j - t * p.tile_blocks) * kBN;
    }
    return s.kv_base + p.L_v + (j - s.nvid) * kBN;
  } else {
    return s.kv_base + (s.qb - j) * kBN;
  }
}

// Valid column range [lo, hi) of block j for query row r, or false when the
// block needs no mask.
template <Mode M>
__device__ __forceinline__ bool seq_mask(const FwdParams& p, const KvSeq& s, int j,
                                         int r, int& lo, int& hi) {
  if constexpr (M != Mode::kSwa) {
    if (j < s.nvid) return false;
    const int col0 = (j - s.nvid) * kBN;
    if (col0 + kBN <= p.text_len) return false;
    lo = 0;
    hi = p.text_len - col0;
    return true;
  } else {
    const int kb = s.qb - j;
    const bool edge = kb * kBN < s.qb * kBN + (kBN - 1) - p.window + 1;
    if (kb != s.qb && !edge) return false;
    const int qi = s.qb * kBN + r;                 // query position
    const int first = qi - p.window + 1 - kb * kBN;  // lowest allowed column
    const int last = qi - kb * kBN;                // highest allowed column
    lo = first < 0 ? 0 : first;
    hi = last + 1 > kBN ? kBN : last + 1;
    return true;
  }
}

__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(a, parity)) return true;
    if ((it & 255u) == 255u && globaltimer_ns() - t0 > 200000000ull) {
      raise_error(1u);
      return false;
    }
  }
}

// Loads one 64-column panel (128 rows x 128 bytes, 128-byte swizzle) of the
// 128-row block whose first row in the tile-ordered view is `row`.
// Tile-ordered tensors and the text block: rows of the 2-D [B*heads*S, d]
// view.  Video blocks of raster-ordered tensors (R): the block is a box of its
// tile in the (d, W, H, T, slice) view, landing in shared memory in the
// tile's own (t, h, w) order.
template <int D, bool R>
__device__ __forceinline__ void load_panel(uint8_t* dst, const CUtensorMap* m2,
                                           const CUtensorMap* m5, uint64_t* bar, int row,
                                           const FwdParams& p, uint64_t pol, int pn) {
  if constexpr (R) {
    const RasterGeom& g = p.rg;
    const int slice = row / g.S;
    const int off = row - slice * g.S;
    if (off < p.L_v) {
      const int tile = off / p.V;
      const int ins = off - tile * p.V;
      const int it = ins / (g.ch * g.cw);
      const int ih = (ins / g.cw) % g.ch;
      const int tw = tile % g.NW;
      const int th = (tile / g.NW) % g.NH;
      const int tt = tile / (g.NW * g.NH);
      tma_load_5d(dst + pn * 128 * 128, m5, bar, pn * 64, tw * g.cw, th * g.ch + ih,
                  tt * g.ct + it, slice, pol);
      return;
    }
  }
  tma_load_2d_hint(dst + pn * 128 * 128, m2, bar, pn * 64, row, pol);
}

// kSwa3d, tiles with 8 x 8 tokens per t-slice: each 128-key block holds two
// t-slices of 64 keys, one per softmax half.  Bit c of the result is set when
// key c of this thread's half (in-tile order: c = 8*h + w) lies in the token
// window [ws, ws + we) of the query along every axis.
__device__ __forceinline__ uint64_t swa3d_half_mask(int key_t, int key_h0, int key_w0,
                                                    const int ws[3], const int we[3]) {
  if (key_t < ws[0] || key_t >= ws[0] + we[0]) return 0ull;
  auto bits8 = [](int lo, int hi) -> uint32_t {
    lo = lo < 0 ? 0 : (lo > 8 ? 8 : lo);
    hi = hi < 0 ? 0 : (hi > 8 ? 8 : hi);
    return hi > lo ? ((1u << hi) - 1u) & ~((1u << lo) - 1u) : 0u;
  };
  const uint32_t mh = bits8(ws[1] - key_h0, ws[1] + we[1] - key_h0);
  const uint64_t mw = bits8(ws[2] - key_w0, ws[2] + we[2] - key_w0);
  uint64_t m = 0;
#pragma unroll
  for (int ih = 0; ih < 8; ++ih)
    if ((mh >> ih) & 1u) m |= mw << (8 * ih);
  return m;
}

// Raster row of tile-ordered row `row` (identity for text rows).
__device__ __forceinline__ int raster_row(const FwdParams& p, int row) {
  const RasterGeom& g = p.rg;
  const int slice = row / g.S;
  const int off = row - slice * g.S;
  if (off >= p.L_v) return row;
  const int tile = off / p.V;
  const int ins = off - tile * p.V;
  const int it = ins / (g.ch * g.cw);
  const int ih = (ins / g.cw) % g.ch;
  const int iw = ins % g.cw;
  const int tw = tile % g.NW;
  const int th = (tile / g.NW) % g.NH;
  const int tt = tile / (g.NW * g.NH);
  return slice * g.S + ((tt * g.ct + it) * g.H + th * g.ch + ih) * g.W + tw * g.cw + iw;
}

// S_slot = Q_slot K^T over d (SS; K block in stage ks) into the score
// buffer at TMEM column scol.  All operands warp-uniform, accumulate flags
// constant.
template <int D, int SLOT>
__device__ __forceinline__ void fwd_issue_s(uint32_t tm, uint64_t dq, uint64_t dk, int ks,
                                            uint32_t scol) {
  using C = FwdCfg<D>;
  constexpr uint32_t kIdesc = idesc_bf16(kBM, kBN, false);
  const uint64_t qa = dq + ((SLOT * C::kBlockBytes) >> 4);
  const uint64_t ka = dk + ((static_cast<uint32_t>(ks) * C::kBlockBytes) >> 4);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = ((kk >> 2) * C::kPanelBytes + (kk & 3) * 32) >> 4;
    umma_ss(tm + scol, qa + off, ka + off, kIdesc, kk > 0 ? 1u : 0u);
  }
}

// O_slot (+)= P_slot V (TS: P from the score buffer at TMEM column pcol, V
// block in stage vs as an MN-major operand, N = d).  P of the keys served by
// softmax column group g (128 / kSplit keys each) sits in the first half of
// that group's own score columns: keys 16 kk .. 16 kk + 15 at column
// (kk / G) * 128 / kSplit + (kk % G) * 8 of the buffer, G = 8 / kSplit
// k-steps per group.
template <int D, int SLOT, bool ACC>
__device__ __forceinline__ void fwd_issue_pv(uint32_t tm, uint64_t dv, int vs, uint32_t pcol) {
  using C = FwdCfg<D>;
  constexpr uint32_t kIdesc = idesc_bf16(kBM, D, true);
  constexpr int G = (kBN / 16) / kSplit;
  const uint64_t va = dv + ((static_cast<uint32_t>(vs) * C::kBlockBytes) >> 4);
#pragma unroll
  for (int kk = 0; kk < kBN / 16; ++kk) {
    const uint32_t acol = (kk / G) * (kBN / kSplit) + (kk % G) * 8;
    umma_ts(tm + C::kOCol + SLOT * D, tm + pcol + acol, va + ((kk * 16 * 128) >> 4), kIdesc,
            (ACC || kk > 0) ? 1u : 0u);
  }
}

template <int D, Mode M, bool R>
__global__ void __launch_bounds__(kFwdThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmap_q,
                    const __grid_constant__ CUtensorMap tmap_k,
                    const __grid_constant__ CUtensorMap tmap_v,
                    const __grid_constant__ CUtensorMap tmap_q5,
                    const __grid_constant__ CUtensorMap tmap_k5,
                    const __grid_constant__ CUtensorMap tmap_v5,
                    const FwdParams p) {
  using C = FwdCfg<D>;
  constexpr int KST = C::kKStages;
  constexpr int VST = C::kVStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* q_full = bars;
  uint64_t* k_full = q_full + 1;
  uint64_t* k_empty = k_full + KST;
  uint64_t* v_full = k_empty + KST;
  uint64_t* v_empty = v_full + VST;
  // s_full / p_full: scores / P of a slot's block in TMEM, [slot] (d = 128)
  // or [slot][block parity] (score-buffer pool, d = 64: a slot's softmax
  // warps may then be a block apart, and two barriers keep the arrivals of
  // neighbouring blocks apart)
  uint64_t* s_full = v_empty + VST;   // [4]
  uint64_t* p_full = s_full + 4;      // [4]
  uint64_t* o_full = p_full + 4;      // [2]
  uint64_t* pv_done = o_full + 2;     // [2] (pool) one more P V of the slot done
  uint64_t* mma_done = pv_done + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const WorkItem item = p.items[blockIdx.x];
  const bool two = item.q1 >= 0;
  const KvSeq seq = make_seq<M>(p, item);
  const int n = seq.n;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    // with the score-buffer pool each slot's Q K^T releases its key stage
    const int k_users = (C::kSBuf == 3 && two) ? 2 : 1;
    for (int i = 0; i < KST; ++i) { mbar_init(&k_full[i], 1); mbar_init(&k_empty[i], k_users); }
    for (int i = 0; i < VST; ++i) { mbar_init(&v_full[i], 1); mbar_init(&v_empty[i], 1); }
    for (int i = 0; i < 4; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 4 * kSplit);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&o_full[i], 1);
      mbar_init(&pv_done[i], 1);
    }
    mbar_init(mma_done, 1);
    bool bad = false;
    if constexpr (STA_DEBUG) bad = !dbg_ok(item_in_bounds<M>(p, item));
    *abort_flag = (error_raised() || n <= 0 || bad) ? 1 : 0;
    fence_mbar_init();
  }
  if (warp == kWarpTma && lane == 0) {
    tma_prefetch_desc(&tmap_q);
    tma_prefetch_desc(&tmap_k);
    tma_prefetch_desc(&tmap_v);
    if constexpr (R) {
      tma_prefetch_desc(&tmap_q5);
      tma_prefetch_desc(&tmap_k5);
      tma_prefetch_desc(&tmap_v5);
    }
  }
  if (warp == kWarpMma) tmem_alloc(tmem_holder, C::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const bool skip = *abort_flag != 0;

  const uint32_t smem_q = smem_u32(smem + C::kQOff);
  const uint32_t smem_k = smem_u32(smem + C::kKOff);
  const uint32_t smem_v = smem_u32(smem + C::kVOff);

  if (warp == kWarpTma) {
    // ------------------------------------------------------------ producer
    // A thread's TMA loads complete one after another, so each operand panel
    // has its own lane: lanes 0 .. kPanels-1 load the key panels, lanes
    // kPanels .. 2 kPanels-1 the value panels (and the first ones the query
    // blocks); the panel-0 lane of each operand posts the expected bytes.
    constexpr int kPanels = C::kPanels;
    if (lane < 2 * kPanels && !skip) {
      const bool is_v = lane >= kPanels;
      const int pn = lane % kPanels;
      const uint64_t pol_kv = policy_evict_last();
      const uint64_t pol_q = policy_evict_first();
      const bool drop_q = *reinterpret_cast<volatile int*>(&g_inject) == 1;
      if (!drop_q) {
        if (lane == 0) mbar_arrive_expect_tx(q_full, (two ? 2 : 1) * C::kBlockBytes);
        const int s = is_v ? 1 : 0;      // key lanes load slot 0, value lanes slot 1
        if (s == 0 || two)
          load_panel<D, R>(smem + C::kQOff + s * C::kBlockBytes, &tmap_q, &tmap_q5, q_full,
                           s ? item.q1 : item.q0, p, pol_q, pn);
      }
      uint64_t* full = is_v ? v_full : k_full;
      uint64_t* empty = is_v ? v_empty : k_empty;
      constexpr int NST = KST;           // key and value rings have the same depth
      static_assert(KST == VST, "one ring depth for both operands");
      const CUtensorMap* m2 = is_v ? &tmap_v : &tmap_k;
      const CUtensorMap* m5 = is_v ? &tmap_v5 : &tmap_k5;
      uint8_t* base = smem + (is_v ? C::kVOff : C::kKOff);
      for (int j = 0; j < n; ++j) {
        const int st = j % NST;
        if (j >= NST && !mbar_wait(&empty[st], ((j / NST) - 1) & 1, abort_flag)) break;
        const int row = seq_row<M>(p, seq, j);
        if (!dbg_ok(row >= 0 && row + kBN <= p.dbg_rows_kv)) {
          *abort_flag = 1;                 // the other roles give up at their next poll
          break;
        }
        if (pn == 0) mbar_arrive_expect_tx(&full[st], C::kBlockBytes);
        load_panel<D, R>(base + st * C::kBlockBytes, m2, m5, &full[st], row, p, pol_kv, pn);
      }
      __syncwarp((1u << (2 * kPanels)) - 1u);
      // Leave no copy in flight: wait for the last load of every stage.
      if (lane == 0) {
        if (!drop_q) mbar_wait_drain(q_full, 0);
        for (int st = 0; st < NST && st < n; ++st) {
          const int last = st + ((n - 1 - st) / NST) * NST;
          mbar_wait_drain(&k_full[st], (last / NST) & 1);
          mbar_wait_drain(&v_full[st], (last / NST) & 1);
        }
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop and waits; one elected lane issues (the
    // same lane every time, so the MMAs and commits keep their issue order).
    if (!skip) {
      const uint32_t tm = warp_uniform(tmem);
      // descriptor bases; per-MMA offsets go into the address field (bytes >> 4)
      const uint64_t dq = sdesc_sw128(warp_uniform(smem_q), 16, 1024);
      const uint64_t dk = sdesc_sw128(warp_uniform(smem_k), 16, 1024);
      const uint64_t dv = sdesc_sw128(warp_uniform(smem_v), C::kPanelBytes, 1024);
      bool ok = mbar_wait_warp(q_full, 0, abort_flag) && mbar_wait_warp(&k_full[0], 0, abort_flag);
      if constexpr (C::kSBuf == 3) {
        // Pool of three score buffers: the scores of slot s, block j go to
        // buffer (2 j + s) % 3.  S1(j+1) takes the buffer P0(j) leaves once
        // P0 V is issued, S0(j+2) the one P1(j) leaves, so each slot's next
        // scores are computed while its softmax of the current block runs.
        auto col = [](int j, int s) { return static_cast<uint32_t>(((2 * j + s) % 3) * 128); };
        if (ok) {
          tc_fence_after();
          if (elect_one()) {
            fwd_issue_s<D, 0>(tm, dq, dk, 0, 0u);
            umma_commit(&s_full[0]);
            umma_commit(&k_empty[0]);
            if (two) {
              fwd_issue_s<D, 1>(tm, dq, dk, 0, 128u);
              umma_commit(&s_full[2]);
              umma_commit(&k_empty[0]);
            }
          }
          __syncwarp();
          if (n > 1) {
            ok = mbar_wait_warp(&k_full[1 % KST], (1 / KST) & 1, abort_flag);
            if (ok) {
              tc_fence_after();
              if (elect_one()) {
                fwd_issue_s<D, 0>(tm, dq, dk, 1 % KST, 256u);
                umma_commit(&s_full[1]);
                umma_commit(&k_empty[1 % KST]);
              }
              __syncwarp();
            }
          }
        }
        for (int j = 0; ok && j < n; ++j) {
          const int vs = j % VST;
          if (!mbar_wait_warp(&v_full[vs], (j / VST) & 1, abort_flag)) break;
          if (!mbar_wait_warp(&p_full[j & 1], (j >> 1) & 1, abort_flag)) break;
          tc_fence_after();
          if (elect_one()) {
            const uint32_t pc = col(j, 0);
            if (j > 0) fwd_issue_pv<D, 0, true>(tm, dv, vs, pc);
            else fwd_issue_pv<D, 0, false>(tm, dv, vs, pc);
            umma_commit(&pv_done[0]);
            if (j == n - 1) umma_commit(&o_full[0]);
          }
          __syncwarp();
          if (two) {
            if (j + 1 < n) {
              const int ks = (j + 1) % KST;
              if (!mbar_wait_warp(&k_full[ks], ((j + 1) / KST) & 1, abort_flag)) break;
              tc_fence_after();
              if (elect_one()) {
                fwd_issue_s<D, 1>(tm, dq, dk, ks, col(j + 1, 1));
                umma_commit(&s_full[2 + ((j + 1) & 1)]);
                umma_commit(&k_empty[ks]);
              }
              __syncwarp();
            }
            if (!mbar_wait_warp(&p_full[2 + (j & 1)], (j >> 1) & 1, abort_flag)) break;
            tc_fence_after();
            if (elect_one()) {
              const uint32_t pc = col(j, 1);
              if (j > 0) fwd_issue_pv<D, 1, true>(tm, dv, vs, pc);
              else fwd_issue_pv<D, 1, false>(tm, dv, vs, pc);
              umma_commit(&pv_done[1]);
              if (j == n - 1) umma_commit(&o_full[1]);
            }
            __syncwarp();
          }
          if (j + 2 < n) {
            const int ks = (j + 2) % KST;
            if (!mbar_wait_warp(&k_full[ks], ((j + 2) / KST) & 1, abort_flag)) break;
            tc_fence_after();
            if (elect_one()) {
              fwd_issue_s<D, 0>(tm, dq, dk, ks, col(j + 2, 0));
              umma_commit(&s_full[(j + 2) & 1]);
              umma_commit(&k_empty[ks]);
            }
            __syncwarp();
          }
          if (elect_one()) umma_commit(&v_empty[vs]);
          __syncwarp();
        }
      } else if (ok) {
        tc_fence_after();
        if (elect_one()) {
          fwd_issue_s<D, 0>(tm, dq, dk, 0, 0u);
          umma_commit(&s_full[0]);
          if (two) {
            fwd_issue_s<D, 1>(tm, dq, dk, 0, 128u);
            umma_commit(&s_full[2]);
          }
          umma_commit(&k_empty[0]);
        }
        __syncwarp();
        for (int j = 0; j < n; ++j) {
          const int vs = j % VST;
          const int jn = j + 1;
          const int ksn = jn % KST;
          // V arrives long before P: wait for it first, so the wait for P
          // is the last thing between the softmax and the P.V MMA
          if (!mbar_wait_warp(&v_full[vs], (j / VST) & 1, abort_flag)) break;
          if (!mbar_wait_warp(&p_full[0], j & 1, abort_flag)) break;
          tc_fence_after();
          if (elect_one()) {
            if (j > 0) fwd_issue_pv<D, 0, true>(tm, dv, vs, 0u);
            else fwd_issue_pv<D, 0, false>(tm, dv, vs, 0u);
          }
          __syncwarp();
          if (jn < n) {
            if (!mbar_wait_warp(&k_full[ksn], (jn / KST) & 1, abort_flag)) break;
            tc_fence_after();
            if (elect_one()) {
              fwd_issue_s<D, 0>(tm, dq, dk, ksn, 0u);
              umma_commit(&s_full[0]);
            }
          } else if (elect_one()) {
            umma_commit(&o_full[0]);
          }
          __syncwarp();
          if (two) {
            if (!mbar_wait_warp(&p_full[2], j & 1, abort_flag)) break;
            tc_fence_after();
            if (elect_one()) {
              if (j > 0) fwd_issue_pv<D, 1, true>(tm, dv, vs, 128u);
              else fwd_issue_pv<D, 1, false>(tm, dv, vs, 128u);
              if (jn < n) {
                fwd_issue_s<D, 1>(tm, dq, dk, ksn, 128u);
                umma_commit(&s_full[2]);
              } else {
                umma_commit(&o_full[1]);
              }
            }
            __syncwarp();
          }
          if (elect_one()) {
            umma_commit(&v_empty[vs]);
            if (jn < n) umma_commit(&k_empty[ksn]);
          }
          __syncwarp();
        }
      }
      // No MMA may still run when TMEM is released.
      if (elect_one()) umma_commit(mma_done);
      __syncwarp();
      mbar_wait_drain(mma_done, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax
    // Warp k of the softmax warps serves slot k / 8, TMEM lane quarter
    // warp % 4 and, in it, the 16 rows of row half (k / 4) % 2; lanes t and
    // t + 16 share row t % 16, lane t + 16 taking columns 64-127 (the
    // .16x32bx2 TMEM accesses), so the two halves of a row meet through a
    // warp shuffle.
    constexpr int kCols = kBN / kSplit;       // score columns per thread
    constexpr int kOCols = D / kSplit;        // output columns per thread
    const int ks = warp - kWarpSoftmax0;
    const int slot = ks / 8;
    const int rh = (ks / 4) % 2;              // row half of the lane quarter
    const int half = lane >> 4;               // column half of the row
    const int sub = warp & 3;                 // TMEM lane quarter of this warp
    const int r = sub * 32 + rh * 16 + (lane & 15);   // query row inside the block
    if (!skip && (slot == 0 || two)) {
      const uint32_t lane_off = static_cast<uint32_t>(sub * 32 + rh * 16) << 16;
      // this warp's 16 lanes; the column half follows from the split offset
      // score buffer of this slot (with the d = 64 pool it changes per block)
      const uint32_t t_s0 = tmem + lane_off;
      const uint32_t t_o = tmem + lane_off + C::kOCol + (slot ? D : 0);
      const float sl2 = p.scale_log2;
      float m_run = -INFINITY;   // running max, log2 units of the scaled scores
      float l_run = 0.f;         // this thread's part of the row sum
      bool done = true;
      // kSwa3d: this query's token window (video rows only)
      bool tok_row = false;
      int tws[3] = {0, 0, 0}, twe[3] = {0, 0, 0};
      if constexpr (M == Mode::kSwa3d) {
        const int off = (slot ? item.q1 : item.q0) + r - item.kv_base;
        if (off < p.L_v) {
          const RasterGeom& g = p.rg;
          const int tile = off / p.V;
          const int ins = off - tile * p.V;
          const int tw = tile % g.NW, th = (tile / g.NW) % g.NH, tt = tile / (g.NW * g.NH);
          const int tok[3] = {tt * g.ct + ins / (g.ch * g.cw), th * g.ch + (ins / g.cw) % g.ch,
                              tw * g.cw + ins % g.cw};
          const int dim[3] = {g.T, g.H, g.W};
#pragma unroll
          for (int a = 0; a < 3; ++a) {
            twe[a] = p.win3[a] < dim[a] ? p.win3[a] : dim[a];
            int st = tok[a] - twe[a] / 2;
            st = st < 0 ? 0 : (st > dim[a] - twe[a] ? dim[a] - twe[a] : st);
            tws[a] = st;
          }
          tok_row = true;
        }
      }
      (void)tok_row;
      // kSlide2d: this query's w x w window
      int sxlo = 0, sylo = 0, swe = 0;
      if constexpr (M == Mode::kSlide2d) {
        const int qpos = (slot ? item.q1 : item.q0) + r - item.kv_base;
        const uint32_t qc = p.coords[qpos];
        swe = p.win2 < p.grid_n ? p.win2 : p.grid_n;
        sxlo = static_cast<int>(qc & 0xffff) - swe / 2;
        sxlo = sxlo < 0 ? 0 : (sxlo > p.grid_n - swe ? p.grid_n - swe : sxlo);
        sylo = static_cast<int>(qc >> 16) - swe / 2;
        sylo = sylo < 0 ? 0 : (sylo > p.grid_n - swe ? p.grid_n - swe : sylo);
      }
      for (int j = 0; j < n; ++j) {
        // barrier of this slot (and, with the pool, of this block's parity)
        const int bi = C::kSBuf == 3 ? 2 * slot + (j & 1) : 2 * slot;
        const uint32_t bph = C::kSBuf == 3 ? (j >> 1) & 1 : j & 1;
        if (!mbar_wait_warp(&s_full[bi], bph, abort_flag)) { done = false; break; }
        tc_fence_after();
        const uint32_t scol = C::kSBuf == 3 ? static_cast<uint32_t>(((2 * j + slot) % 3) * 128)
                                            : (slot ? 128u : 0u);
        const uint32_t t_s = t_s0 + scol;
        // P over the first half of this thread's own score columns, so no
        // thread overwrites scores that another has still to read
        const uint32_t t_p = t_s;
        float s[kCols];
        // this thread's raw scores of block j, masked (called again by the
        // rare recompute below: the scores stay in TMEM until P is stored)
        auto load_scores = [&]() {
          uint32_t sr[kCols];
#pragma unroll
          for (int cc = 0; cc < kCols / 32; ++cc) tmem_ld_half32<kCols>(t_s + cc * 32, sr + cc * 32);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < kCols; ++c) s[c] = __uint_as_float(sr[c]);
          int lo, hi;
          if (seq_mask<M>(p, seq, j, r, lo, hi)) {
            lo -= half * kCols;
            hi -= half * kCols;
  #pragma unroll
            for (int c = 0; c < kCols; ++c)
              if (c < lo || c >= hi) s[c] = -INFINITY;
          }
          if constexpr (M == Mode::kSlide2d) {
            // per-element 2-D window test against the keys' grid coordinates
            const uint4* kc = reinterpret_cast<const uint4*>(
                p.coords + static_cast<size_t>(seq.ids[j]) * kBN + half * kCols);
  #pragma unroll
            for (int c4 = 0; c4 < kCols / 4; ++c4) {
              const uint4 v4 = __ldg(kc + c4);
              const uint32_t cv[4] = {v4.x, v4.y, v4.z, v4.w};
  #pragma unroll
              for (int e = 0; e < 4; ++e) {
                const uint32_t dx = (cv[e] & 0xffffu) - static_cast<uint32_t>(sxlo);
                const uint32_t dy = (cv[e] >> 16) - static_cast<uint32_t>(sylo);
                if (dx >= static_cast<uint32_t>(swe) || dy >= static_cast<uint32_t>(swe))
                  s[c4 * 4 + e] = -INFINITY;
              }
            }
          }
          if constexpr (M == Mode::kSwa3d) {
            static_assert(kSplit == 2, "the 3-D window mask gives each half one t-slice");
            if (tok_row && j < seq.nvid) {
              const RasterGeom& g = p.rg;
              const int kt = j / p.tile_blocks;
              const int sb = j - kt * p.tile_blocks;
              const int kid = seq.ids[kt];
              const int ktw = kid % g.NW, kth = (kid / g.NW) % g.NH, ktt = kid / (g.NW * g.NH);
              const uint64_t km = swa3d_half_mask(ktt * g.ct + sb * 2 + half, kth * g.ch,
                                                  ktw * g.cw, tws, twe);
  #pragma unroll
              for (int c = 0; c < kCols; ++c)
                if (!((km >> c) & 1ull)) s[c] = -INFINITY;
            }
          }
        };
        load_scores();
        // exp2(s * sl2 - ref) two at a time, packed to bf16 as they come
        // (most pairs on the ex2 unit, a fixed share on the FMA pipe); with
        // kMax the raw maximum is taken on the way
        uint32_t pk[kCols / 2];
        auto exp_pack = [&](float ref, auto with_max, float& mx) {
          const float2 sl2v = make_float2(sl2, sl2);
          const float neg = (ref == -INFINITY) ? 0.f : -ref;
          const float2 npv = make_float2(neg, neg);
          float2 ls = make_float2(0.f, 0.f);
          float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
          for (int c = 0; c < kCols; c += 2) {
            if constexpr (decltype(with_max)::value) {
              if ((c & 2) == 0) m0 = fmax3(m0, s[c], s[c + 1]);
              else m1 = fmax3(m1, s[c], s[c + 1]);
            }
            const float2 x = __ffma2_rn(make_float2(s[c], s[c + 1]), sl2v, npv);
            float2 e;
            if (exp2_on_fma(c / 2)) {   // resolved at compile time (unrolled)
              e = exp2_fma2(x);
            } else {
              e = make_float2(fast_exp2(x.x), fast_exp2(x.y));
            }
            ls = __fadd2_rn(ls, e);
            pk[c / 2] = pack_bf16x2(e.x, e.y);
          }
          if constexpr (decltype(with_max)::value) mx = fmaxf(m0, m1);
          return ls.x + ls.y;
        };
        // row max: four independent chains of three-input max
        auto own_max = [&]() {
          constexpr int kQ = kCols / 4;
          float mq[4];
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            float m = s[k4 * kQ];
#pragma unroll
            for (int i = 1; i + 1 < kQ; i += 2) m = fmax3(m, s[k4 * kQ + i], s[k4 * kQ + i + 1]);
            if constexpr (kQ % 2 == 0) m = fmaxf(m, s[k4 * kQ + kQ - 1]);
            mq[k4] = m;
          }
          return fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
        };
        // the halves of a row (lanes t, t + 16) agree on the block's max
        auto exchange_max = [&](float& mx) {
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
          return true;
        };
        // Reference of the exponent: the running max (log2 units), raised
        // only when the block's max exceeds it by more than 2^8.  Rows that
        // have a running max take the exponentials against it at once and
        // the block's max on the way; in the rare case that max raises the
        // reference, the block is recomputed from its scores in TMEM.  A warp
        // with a row that has no running max yet (its first unmasked block)
        // agrees on the max first.  Both halves of a row see the same rows'
        // state, so they take the same branches.
        using kNoMax = std::integral_constant<bool, false>;
        using kWithMax = std::integral_constant<bool, true>;
        float mx = -INFINITY;
        float lsum;
        bool resc;
        float alpha = 1.f;
        if (__any_sync(0xffffffffu, m_run == -INFINITY)) {
          mx = own_max();
          if (!exchange_max(mx)) { done = false; break; }
          const float m_cand = mx * sl2;
          resc = m_cand > m_run + 8.0f;
          if (resc) {
            alpha = fast_exp2(m_run - m_cand);
            m_run = m_cand;
            l_run *= alpha;
          }
          lsum = exp_pack(m_run, kNoMax{}, mx);
        } else {
          lsum = exp_pack(m_run, kWithMax{}, mx);
          if (!exchange_max(mx)) { done = false; break; }
          const float m_cand = mx * sl2;
          resc = m_cand > m_run + 8.0f;
          if (resc) {
            alpha = fast_exp2(m_run - m_cand);
            m_run = m_cand;
            l_run *= alpha;
          }
          if (__any_sync(0xffffffffu, resc)) {
            load_scores();
            lsum = exp_pack(m_run, kNoMax{}, mx);
          }
        }
        // bf16 P over the first half of this thread's own score columns
#pragma unroll
        for (int cc = 0; cc < kCols / 32; ++cc) tmem_st_half16<kCols>(t_p + cc * 16, pk + cc * 16);
        l_run += lsum;
        if (j > 0 && __any_sync(0xffffffffu, resc)) {
          if constexpr (C::kSBuf == 3) {
            // the pool lets this block's scores come before the previous
            // block's P V: wait until that has landed in O
            if (!mbar_wait_warp(&pv_done[slot], (j - 1) & 1, abort_flag)) { done = false; break; }
            tc_fence_after();
          }
#pragma unroll
          for (int cc = 0; cc < kOCols / 32; ++cc) {
            uint32_t o[32];
            tmem_ld_half32<kOCols>(t_o + cc * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st_half32<kOCols>(t_o + cc * 32, o);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[bi]);
      }
      if (done && mbar_wait_warp(&o_full[slot], 0, abort_flag)) {
        tc_fence_after();
        l_run += __shfl_xor_sync(0xffffffffu, l_run, 16);
        {
          const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
          int qrow = (slot ? item.q1 : item.q0) + r;
          if constexpr (R) qrow = raster_row(p, qrow);
          const bool row_ok = dbg_ok(qrow >= 0 && qrow < p.dbg_rows_q);
          if (!row_ok) qrow = 0;             // debug build: the stores below are skipped
          uint4* dst = reinterpret_cast<uint4*>(p.out + static_cast<size_t>(qrow) * D +
                                                half * kOCols);
#pragma unroll
          for (int cc = 0; cc < kOCols / 32; ++cc) {
            uint32_t o[32];
            tmem_ld_half32<kOCols>(t_o + cc * 32, o);
            tmem_wait_ld();
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e)
              pk[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv,
                                  __uint_as_float(o[2 * e + 1]) * inv);
            if (row_ok) {
#pragma unroll
              for (int v4 = 0; v4 < 4; ++v4)
                dst[cc * 4 + v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2],
                                              pk[4 * v4 + 3]);
            }
          }
          if (p.lse != nullptr && half == 0 && row_ok) {
            const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
            p.lse[qrow] = (m_use + __log2f(l_run)) * 0.69314718055994531f;
          }
        }
      }
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace sta
