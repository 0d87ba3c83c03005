// attn_fwd_pair.cuh - STA forward for d = 128 on a pair of SMs (cta_group::2).
//
// Same computation as attn_fwd_kernel<128, Mode::kSta, R> (STA README,
// "Usage" and "Why is STA Fast?": dense 128-key blocks of whole key tiles,
// only the padded text block masked), scheduled for Blackwell's paired MMA:
//
//  * A cluster of two CTAs takes one work item: two 128-row query blocks
//    with the same key-block list, one block per CTA.  Every Q K^T and P V
//    is one tcgen05.mma.cta_group::2 with M = 256 (128 rows per SM), issued
//    by the even CTA.  Its B operand is split along N between the two SMs:
//    each CTA loads half of every key block (64 keys, all of d) for Q K^T and
//    half of d (all 128 keys) of every value block for P V, so each SM moves
//    half the K / V bytes through its shared memory.
//  * One query block per SM leaves TMEM room for three score buffers next to
//    the O accumulator: S(j+1) and S(j+2) are computed while the softmax of
//    block j runs, so the softmax never waits for the MMA round trip.
//  * Two softmax groups of 8 warps alternate key blocks (group j % 2 takes
//    block j); two warps share a query row, 64 scores each.  The exponent
//    reference of block j is the running max after block j (raised only when
//    a row's max grows by more than 2^8), handed from group to group through
//    shared memory.  When it grows, the group rescales O after P_{j-1} V has
//    landed and before P_j V is issued; each group keeps its own partial row
//    sums, merged in the epilogue.
//
// Warps (both CTAs): 0 key and query loads, 18 value loads (several lanes,
// each an independent stream of TMA loads), 1 MMA issuer (even CTA; the odd
// CTA's warp 1 only takes part in the TMEM allocation), 2-9 softmax group 0,
// 10-17 softmax group 1.  TMEM (512 columns, both SMs): S0, S1, S2 at 0, 128,
// 256; O at 384.  P_j is written, as bf16, over the first half of each
// warp's own 64 score columns of S_{j % 3}.
//
// Every wait is bounded (device_ptx.cuh); a CTA that gives up records the
// device error word, and all paths still meet the final cluster barrier, so
// neither CTA leaves while the other may still signal its barriers.
#pragma once

#include "attn_fwd.cuh"

namespace sta {

struct PairCfg {
  static constexpr int D = 128;
  static constexpr int kQPanel = 128 * 128;          // 128 rows x 128 B
  static constexpr int kQBytes = 2 * kQPanel;        // own query block
  static constexpr int kKPanel = 64 * 128;           // 64 keys x 128 B
  static constexpr int kKBytes = 2 * kKPanel;        // half a key block, all of d
  static constexpr int kVBytes = 128 * 128;          // 128 keys x this CTA's 64 columns
  static constexpr int KST = 5;                      // key stages
  static constexpr int VST = 5;                      // value stages
  static constexpr int SB = 3;                       // score buffers
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + kQBytes;
  static constexpr int kVOff = kKOff + KST * kKBytes;
  static constexpr int kBarOff = kVOff + VST * kVBytes;
  static constexpr int kBarBytes = 512;
  static constexpr int kRedOff = kBarOff + kBarBytes;
  // floats: max exchange [group][parity][half][128], reference hand-off
  // [parity][128], epilogue sums [item parity][group][half][128] and
  // references [item parity][group][128]
  static constexpr int kRedFloats = 2 * 2 * 2 * 128 + 2 * 128 + 2 * (2 * 2 * 128 + 2 * 128);
  static constexpr int kSmemBytes = kRedOff + kRedFloats * 4 + 1024;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kOCol = 384;
};

// warps: 0 key and query loads, 1 MMA, 2-17 softmax, 18 value loads
constexpr int kWarpKLoad = 0;
constexpr int kWarpVLoad = 18;
constexpr int kLoadStreams = 4;   // load streams (lanes) per operand panel
// A stream waits for the release of the stage it is about to fill by phase
// parity, which is only unambiguous while the stream is at most one phase
// ahead of that stage's barrier.  With more streams than stages a stream can
// reach block g + streams while block g (same stage, another phase) has not
// even landed, pass the parity wait early and load into a stage in use.
static_assert(kLoadStreams <= PairCfg::KST && kLoadStreams <= PairCfg::VST,
              "at most one load stream per ring stage");
constexpr int kPairThreads = 19 * 32;

// Q K^T into score buffer `b` (SS pair MMA, M = 256, N = 128 keys, K = d).
__device__ __forceinline__ void pair_issue_s(uint32_t tm, uint64_t dq, uint64_t dk, int b,
                                             int ks) {
  using C = PairCfg;
  constexpr uint32_t kIdesc = idesc_bf16(256, 128, false);
  const uint64_t ka = dk + ((static_cast<uint32_t>(ks) * C::kKBytes) >> 4);
  const uint32_t d = tm + static_cast<uint32_t>(b) * 128u;
#pragma unroll
  for (int kk = 0; kk < C::D / 16; ++kk) {
    const uint32_t qo = ((kk >> 2) * C::kQPanel + (kk & 3) * 32) >> 4;
    const uint32_t ko = ((kk >> 2) * C::kKPanel + (kk & 3) * 32) >> 4;
    umma_ss_pair(d, dq + qo, ka + ko, kIdesc, kk > 0 ? 1u : 0u);
  }
}

// O (+)= P V from score buffer `b` (TS pair MMA, M = 256, N = d, K = 128
// keys; B is each CTA's 64 columns of d, MN-major).  P of keys 0-63 sits in
// columns 0-31 of the buffer, of keys 64-127 in columns 64-95.
template <bool ACC>
__device__ __forceinline__ void pair_issue_pv(uint32_t tm, uint64_t dv, int b, int vs) {
  using C = PairCfg;
  constexpr uint32_t kIdesc = idesc_bf16(256, C::D, true);
  const uint64_t va = dv + ((static_cast<uint32_t>(vs) * C::kVBytes) >> 4);
  const uint32_t pb = tm + static_cast<uint32_t>(b) * 128u;
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint32_t acol = (kk < 4) ? kk * 8 : 64 + (kk - 4) * 8;
    umma_ts_pair(tm + C::kOCol, pb + acol, va + ((kk * 16 * 128) >> 4), kIdesc,
                 (ACC || kk > 0) ? 1u : 0u);
  }
}

// First row and 5-D box origin of one 128-row block; `half` >= 0 selects the
// 64-row half (keys) of the box, split along t when the box spans two or
// more t-slices, else along h.
template <bool R>
__device__ __forceinline__ void pair_load(uint8_t* dst, int panels, int panel0, const CUtensorMap* m2,
                                          const CUtensorMap* m5, uint32_t bar, int row, int half,
                                          const FwdParams& p, uint64_t pol) {
  if constexpr (R) {
    const RasterGeom& g = p.rg;
    const int slice = row / g.S;
    const int off = row - slice * g.S;
    if (off < p.L_v) {
      const int tile = off / p.V;
      const int ins = off - tile * p.V;
      int it = ins / (g.ch * g.cw);
      int ih = (ins / g.cw) % g.ch;
      if (half >= 0) {
        if (p.khalf_t) it += half * p.kbox_t / 2;
        else ih += half * p.kbox_h / 2;
      }
      const int tw = tile % g.NW;
      const int th = (tile / g.NW) % g.NH;
      const int tt = tile / (g.NW * g.NH);
      const int bytes = half >= 0 ? PairCfg::kKPanel : PairCfg::kQPanel;
      for (int pn = 0; pn < panels; ++pn)
        tma_load_5d_pair(dst + pn * bytes, m5, bar, (panel0 + pn) * 64, tw * g.cw,
                         th * g.ch + ih, tt * g.ct + it, slice, pol);
      return;
    }
  }
  const int bytes = half >= 0 ? PairCfg::kKPanel : PairCfg::kQPanel;
  const int r0 = row + (half >= 0 ? half * 64 : 0);
  for (int pn = 0; pn < panels; ++pn)
    tma_load_2d_pair(dst + pn * bytes, m2, bar, (panel0 + pn) * 64, r0, pol);
}

// Items of one cluster: p.items[p.item_off[c] .. p.item_off[c + 1]), cluster
// c of gridDim.x / 2 (persistent: one cluster per pair of SMs, items
// assigned longest first to the least loaded cluster on the host).
__device__ __forceinline__ int pair_item_begin(const FwdParams& p, int c) { return p.item_off[c]; }
__device__ __forceinline__ int pair_item_end(const FwdParams& p, int c) { return p.item_off[c + 1]; }

template <bool R>
__global__ void __launch_bounds__(kPairThreads, 1)
    attn_fwd_pair_kernel(const __grid_constant__ CUtensorMap tmap_q,
                         const __grid_constant__ CUtensorMap tmap_k,
                         const __grid_constant__ CUtensorMap tmap_v,
                         const __grid_constant__ CUtensorMap tmap_q5,
                         const __grid_constant__ CUtensorMap tmap_k5,
                         const __grid_constant__ CUtensorMap tmap_v5,
                         const __grid_constant__ FwdParams p) {
  using C = PairCfg;
  constexpr int KST = C::KST, VST = C::VST, SB = C::SB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  // Every barrier phase below follows a counter that runs across the items of
  // the cluster (item index ii, global block index g), so the pipeline
  // carries on from one item to the next.
  uint64_t* q_full = bars;                 // even CTA: both Q blocks of item ii landed
  uint64_t* q_empty = q_full + 1;          // both: item ii's last Q K^T done
  uint64_t* k_full = q_empty + 1;          // [KST] even CTA: both key halves landed
  uint64_t* v_full = k_full + KST;         // [VST]
  uint64_t* k_empty = v_full + VST;        // [KST] both CTAs: stage free again
  uint64_t* v_empty = k_empty + KST;       // [VST]
  uint64_t* s_full = v_empty + VST;        // [SB] both CTAs: scores of block g ready
  uint64_t* p_full = s_full + SB;          // [SB] even CTA: P of both CTAs written
  // both CTAs: P_g V done, on pv_done[g % 2].  Two barriers so that a group
  // waiting for P_{g-1} V never sees a phase two behind: S_g completing
  // implies P_{g-3} V has completed (one thread's MMAs run in order).
  uint64_t* pv_done = p_full + SB;         // [2]
  uint64_t* o_full = pv_done + 2;          // both CTAs: item ii's last P V done
  uint64_t* o_free = o_full + 1;           // even CTA: O of item ii read (32 warps)
  uint64_t* mma_done = o_free + 1;         // both CTAs: no MMA in flight
  uint64_t* xb = mma_done + 1;             // [2 groups][4 quarters] max exchange
  uint64_t* ref_bar = xb + 8;              // [2 parities] reference hand-off
  uint64_t* sum_bar = ref_bar + 2;         // epilogue sums posted
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sum_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  float* red = reinterpret_cast<float*>(smem + C::kRedOff);   // [2][2][2][128]
  float* ref = red + 2 * 2 * 2 * 128;                          // [2][128]
  float* lsum = ref + 2 * 128;                                 // [2][2][2][128]
  float* msum = lsum + 2 * 2 * 2 * 128;                        // [2][2][128]

  const uint32_t rank = cluster_rank();
  const bool lead = rank == 0;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int cl = static_cast<int>(blockIdx.x >> 1);
  const int it0 = pair_item_begin(p, cl), it1 = pair_item_end(p, cl);

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < KST; ++i) { mbar_init(&k_full[i], 1); mbar_init(&k_empty[i], 1); }
    for (int i = 0; i < VST; ++i) { mbar_init(&v_full[i], 1); mbar_init(&v_empty[i], 1); }
    for (int i = 0; i < SB; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 16);      // 8 softmax warps in each CTA
    }
    mbar_init(&pv_done[0], 1);
    mbar_init(&pv_done[1], 1);
    mbar_init(o_full, 1);
    mbar_init(o_free, 32);            // 16 softmax warps in each CTA
    mbar_init(mma_done, 1);
    for (int i = 0; i < 8; ++i) mbar_init(&xb[i], 2);   // one arrival per warp
    // all 8 warps of the posting group: the half-0 warps after writing the
    // value, the half-1 warps after reading the previous one, so the next
    // writer of the slot cannot overtake a reader
    for (int i = 0; i < 2; ++i) mbar_init(&ref_bar[i], 8);
    mbar_init(sum_bar, 16);
    *abort_flag = (error_raised() || it1 <= it0) ? 1 : 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmap_q);
    tma_prefetch_desc(&tmap_k);
    tma_prefetch_desc(&tmap_v);
    if constexpr (R) {
      tma_prefetch_desc(&tmap_q5);
      tma_prefetch_desc(&tmap_k5);
      tma_prefetch_desc(&tmap_v5);
    }
  }
  if (warp == 1) tmem_alloc_pair(tmem_holder, C::kTmemCols);
  tc_fence_before();
  __syncthreads();
  cluster_sync();          // both CTAs' barriers initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  // one decision for the pair: the even CTA's
  const bool skip =
      (lead ? *abort_flag : static_cast<int>(ld_shared_cluster_u32(
                                map_to_cta(smem_u32(const_cast<int*>(abort_flag)), 0)))) != 0;
  if (!lead && skip) *abort_flag = 1;

  const uint32_t smem_q = smem_u32(smem + C::kQOff);
  const uint32_t smem_k = smem_u32(smem + C::kKOff);
  const uint32_t smem_v = smem_u32(smem + C::kVOff);

  if (warp == kWarpKLoad) {
    // ------------------------------------------------------------ key / query loads
    // A thread's TMA loads complete one after another, so every lane runs
    // its own stream: lanes 0-7 take the key blocks g with g % 4 == lane / 2
    // (panel lane % 2 of d), lanes 8-9 the query block of each item (one
    // panel each).  A slow load then holds up only its own stream.
    if (!skip && lane < 2 * kLoadStreams + 2) {
      const int pn = lane & 1;
      const uint64_t pol_kv = policy_evict_last();
      const uint64_t pol_q = policy_evict_first();
      if (lane < 2 * kLoadStreams) {
        const int si = lane >> 1;
        int g = 0;
        bool ok = true;
        for (int it = it0; ok && it < it1; ++it) {
          const WorkItem item = p.items[it];
          const KvSeq seq = make_seq<Mode::kSta>(p, item);
          for (int j = 0; j < seq.n; ++j, ++g) {
            if (g % kLoadStreams != si) continue;
            const int ks = g % KST;
            if (g >= KST && !mbar_wait(&k_empty[ks], ((g / KST) - 1) & 1, abort_flag)) {
              ok = false;
              break;
            }
            const int row = seq_row<Mode::kSta>(p, seq, j);
            if (lead && pn == 0) mbar_arrive_expect_tx(&k_full[ks], 2 * C::kKBytes);
            pair_load<R>(smem + C::kKOff + ks * C::kKBytes + pn * C::kKPanel, 1, pn, &tmap_k,
                         &tmap_k5, map_to_cta(smem_u32(&k_full[ks]), 0), row,
                         static_cast<int>(rank), p, pol_kv);
          }
        }
      } else if (*reinterpret_cast<volatile int*>(&g_inject) != 1) {
        int ii = 0;
        for (int it = it0; it < it1; ++it, ++ii) {
          const WorkItem item = p.items[it];
          const int qrow = (rank == 1 && item.q1 >= 0) ? item.q1 : item.q0;
          // Q of the previous item is free once its last Q K^T is done
          if (ii > 0 && !mbar_wait(q_empty, (ii - 1) & 1, abort_flag)) break;
          if (lead && pn == 0) mbar_arrive_expect_tx(q_full, 2 * C::kQBytes);
          pair_load<R>(smem + C::kQOff + pn * C::kQPanel, 1, pn, &tmap_q, &tmap_q5,
                       map_to_cta(smem_u32(q_full), 0), qrow, -1, p, pol_q);
        }
      }
    }
    __syncwarp();
    // Leave no copy in flight (normally the MMAs have consumed every load
    // already): the even CTA's full barriers count the bytes of both CTAs.
    if (lead && lane == 0 && !skip) {
      int nb = 0, ni = 0;
      for (int it = it0; it < it1; ++it, ++ni) nb += make_seq<Mode::kSta>(p, p.items[it]).n;
      for (int st = 0; st < KST && st < nb; ++st) {
        const int last = st + ((nb - 1 - st) / KST) * KST;
        mbar_wait_drain(&k_full[st], (last / KST) & 1);
      }
      if (ni > 0 && *reinterpret_cast<volatile int*>(&g_inject) != 1)
        mbar_wait_drain(q_full, (ni - 1) & 1);
    }
  } else if (warp == kWarpVLoad) {
    // ------------------------------------------------------------ value loads
    // lanes 0-3: the value blocks g with g % 4 == lane
    if (!skip && lane < kLoadStreams) {
      const uint64_t pol_kv = policy_evict_last();
      int g = 0;
      bool ok = true;
      for (int it = it0; ok && it < it1; ++it) {
        const WorkItem item = p.items[it];
        const KvSeq seq = make_seq<Mode::kSta>(p, item);
        for (int j = 0; j < seq.n; ++j, ++g) {
          if (g % kLoadStreams != lane) continue;
          const int vs = g % VST;
          if (g >= VST && !mbar_wait(&v_empty[vs], ((g / VST) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          const int row = seq_row<Mode::kSta>(p, seq, j);
          if (lead) mbar_arrive_expect_tx(&v_full[vs], 2 * C::kVBytes);
          pair_load<R>(smem + C::kVOff + vs * C::kVBytes, 1, static_cast<int>(rank), &tmap_v,
                       &tmap_v5, map_to_cta(smem_u32(&v_full[vs]), 0), row, -1, p, pol_kv);
        }
      }
    }
    __syncwarp();
    if (lead && lane == 0 && !skip) {
      int nb = 0;
      for (int it = it0; it < it1; ++it) nb += make_seq<Mode::kSta>(p, p.items[it]).n;
      for (int st = 0; st < VST && st < nb; ++st) {
        const int last = st + ((nb - 1 - st) / VST) * VST;
        mbar_wait_drain(&v_full[st], (last / VST) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Two cursors over the cluster's blocks: Q K^T runs SB blocks ahead of
    // P V (score buffer g % SB is free once P_{g-SB} V has been issued).
    if (lead && !skip) {
      const uint32_t tm = warp_uniform(tmem);
      const uint64_t dq = sdesc_sw128(warp_uniform(smem_q), 16, 1024);
      const uint64_t dk = sdesc_sw128(warp_uniform(smem_k), 16, 1024);
      const uint64_t dv = sdesc_sw128(warp_uniform(smem_v), C::kVBytes, 1024);
      // S cursor: item s_it, block s_j of s_n; s_need_q: its Q not yet waited for
      int s_it = it0 - 1, s_j = 0, s_n = 0, s_ii = -1, gs = 0;
      bool s_need_q = false, s_end = false;
      bool ok = true;
      // Issues Q K^T for the S cursor's next block: 1 issued, 0 not now (the
      // next item's Q has not landed and may_wait is false, or no block
      // left), -1 a wait gave up.
      auto issue_next_s = [&](bool may_wait) -> int {
        if (s_end) return 0;
        if (s_j >= s_n && !s_need_q) {
          // leaving item s_it: its Q is free once this Q K^T completes
          if (s_it >= it0 && elect_one()) umma_commit_pair(q_empty);
          __syncwarp();
          if (++s_it >= it1) {
            s_end = true;
            return 0;
          }
          ++s_ii;
          s_n = make_seq<Mode::kSta>(p, p.items[s_it]).n;
          s_j = 0;
          s_need_q = true;
        }
        if (s_need_q) {
          if (may_wait) {
            if (!mbar_wait_warp(q_full, s_ii & 1, abort_flag)) return -1;
          } else if (!__shfl_sync(0xffffffffu, mbar_test_wait(smem_u32(q_full), s_ii & 1), 0)) {
            return 0;
          }
          s_need_q = false;
        }
        const int ks = gs % KST;
        if (!mbar_wait_warp(&k_full[ks], (gs / KST) & 1, abort_flag)) return -1;
        tc_fence_after();
        if (elect_one()) {
          pair_issue_s(tm, dq, dk, gs % SB, ks);
          umma_commit_pair(&s_full[gs % SB]);
          umma_commit_pair(&k_empty[ks]);
        }
        __syncwarp();
        ++s_j;
        ++gs;
        return 1;
      };
      while (gs < SB) {
        const int r = issue_next_s(true);
        if (r <= 0) {
          ok = r == 0;
          break;
        }
      }
      // P V cursor
      int v_it = it0, v_j = 0, v_ii = 0, gp = 0;
      int v_n = make_seq<Mode::kSta>(p, p.items[it0]).n;
      while (ok) {
        if (v_j >= v_n) {
          if (++v_it >= it1) break;
          ++v_ii;
          v_n = make_seq<Mode::kSta>(p, p.items[v_it]).n;
          v_j = 0;
          // O of the previous item must have been read out
          if (!mbar_wait_warp(o_free, (v_ii - 1) & 1, abort_flag)) break;
        }
        // the scores of this block must be on their way
        while (gs <= gp) {
          const int r = issue_next_s(true);
          if (r <= 0) {
            ok = r == 0 && gs > gp;
            break;
          }
        }
        if (!ok) break;
        const int vs = gp % VST;
        const int b = gp % SB;
        if (!mbar_wait_warp(&v_full[vs], (gp / VST) & 1, abort_flag)) break;
        if (!mbar_wait_warp(&p_full[b], (gp / SB) & 1, abort_flag)) break;
        tc_fence_after();
        if (elect_one()) {
          if (v_j > 0) pair_issue_pv<true>(tm, dv, b, vs);
          else pair_issue_pv<false>(tm, dv, b, vs);
          umma_commit_pair(&v_empty[vs]);
          umma_commit_pair(&pv_done[gp & 1]);
          if (v_j == v_n - 1) umma_commit_pair(o_full);
        }
        __syncwarp();
        ++v_j;
        ++gp;
        // keep Q K^T up to SB blocks ahead, without waiting for a new Q
        while (gs < gp + SB) {
          const int r = issue_next_s(false);
          if (r <= 0) {
            if (r < 0) ok = false;
            break;
          }
        }
      }
      if (elect_one()) umma_commit_pair(mma_done);
      __syncwarp();
    }
    // both CTAs keep their TMEM until the pair's MMAs are done
    if (!skip) mbar_wait_drain(mma_done, 0);
  } else {
    // ------------------------------------------------------------ softmax
    const int sw = warp - 2;
    const int grp = sw >> 3;                  // group: blocks g with g % 2 == grp
    const int half = (sw >> 2) & 1;           // score columns [64 half, 64 half + 64)
    const int sub = warp & 3;                 // TMEM lane quarter
    const int r = sub * 32 + lane;            // row of this CTA's query block
    const uint32_t lane_off = static_cast<uint32_t>(sub * 32) << 16;
    const uint32_t t_o = tmem + lane_off + C::kOCol + half * 64;
    uint64_t* xbg = &xb[grp * 4 + sub];
    const uint32_t pf0 = map_to_cta(smem_u32(p_full), 0);
    const uint32_t of0 = map_to_cta(smem_u32(o_free), 0);
    const float sl2 = p.scale_log2;
    bool done = !skip;
    int gb = 0;                               // global index of the item's block 0
    for (int it = it0, ii = 0; done && it < it1; ++it, ++ii) {
      const WorkItem item = p.items[it];
      const KvSeq seq = make_seq<Mode::kSta>(p, item);
      const int n = seq.n;
      const int qrow = (rank == 1 && item.q1 >= 0) ? item.q1 : item.q0;
      const bool store = rank == 0 || item.q1 >= 0;
      float m_g = -INFINITY;    // reference of this group's partial sum
      float l_g = 0.f;          // partial row sum over this thread's columns
      for (int j = ((gb & 1) == grp) ? 0 : 1; j < n; j += 2) {
        const int g = gb + j;
        const int b = g % SB;
        if (!mbar_wait_warp(&s_full[b], (g / SB) & 1, abort_flag)) { done = false; break; }
        tc_fence_after();
        const uint32_t t_s = tmem + lane_off + b * 128 + half * 64;
        uint32_t sr[64];
        STA_TMEM_LD32(t_s, sr);
        STA_TMEM_LD32(t_s + 32, (sr + 32));
        tmem_wait_ld();
        float s[64];
#pragma unroll
        for (int c = 0; c < 64; ++c) s[c] = __uint_as_float(sr[c]);
        int lo, hi;
        if (seq_mask<Mode::kSta>(p, seq, j, r, lo, hi)) {
          lo -= half * 64;
          hi -= half * 64;
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (c < lo || c >= hi) s[c] = -INFINITY;
        }
        float mq[4];
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
          float m = s[k4 * 16];
#pragma unroll
          for (int i = 1; i + 1 < 16; i += 2) m = fmax3(m, s[k4 * 16 + i], s[k4 * 16 + i + 1]);
          mq[k4] = fmaxf(m, s[k4 * 16 + 15]);
        }
        float mx = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
        // row max over both halves
        const int par = (g >> 1) & 1;
        float* rb = red + ((grp * 2 + par) * 2) * 128;
        rb[half * 128 + r] = mx;
        __syncwarp();
        if (lane == 0) mbar_arrive(xbg);
        if (!mbar_wait_warp(xbg, par, abort_flag)) { done = false; break; }
        mx = fmaxf(mx, rb[(half ^ 1) * 128 + r]);
        // reference after the item's previous block (the other group's).
        // Every block but the cluster's first waits for the previous block's
        // post, even the first block of an item, which does not use it: its
        // own post reuses that slot and barrier, which the previous item's
        // last block may still have to read.
        float m_prev = -INFINITY;
        if (g > 0) {
          if (!mbar_wait_warp(&ref_bar[(g - 1) & 1], ((g - 1) >> 1) & 1, abort_flag)) {
            done = false;
            break;
          }
          if (j > 0) m_prev = ref[((g - 1) & 1) * 128 + r];
        }
        const float m_cand = mx * sl2;
        const float m_use = m_cand > m_prev + 8.0f ? m_cand : m_prev;
        if (half == 0) ref[(g & 1) * 128 + r] = m_use;
        __syncwarp();
        if (lane == 0) mbar_arrive(&ref_bar[g & 1]);
        if (m_g != m_use) {
          l_g = (m_g == -INFINITY) ? 0.f : l_g * fast_exp2(m_g - m_use);
          m_g = m_use;
        }
        const float neg_m = (m_use == -INFINITY) ? 0.f : -m_use;
        float ls0 = 0.f, ls1 = 0.f;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float p0 = fast_exp2(fmaf(s[cc * 32 + 2 * e], sl2, neg_m));
            const float p1 = fast_exp2(fmaf(s[cc * 32 + 2 * e + 1], sl2, neg_m));
            ls0 += p0;
            ls1 += p1;
            pk[e] = pack_bf16x2(p0, p1);
          }
          STA_TMEM_ST16(t_s + cc * 16, pk);
        }
        l_g += ls0 + ls1;
        // O holds blocks < j relative to m_prev: rescale it once P_{g-1} V
        // has landed (P_g V is not issued before this group's arrival
        // below; done after the exponentials, when the scores no longer hold
        // registers)
        if (j > 0 && __any_sync(0xffffffffu, m_use > m_prev)) {
          if (!mbar_wait_warp(&pv_done[(g - 1) & 1], ((g - 1) >> 1) & 1, abort_flag)) {
            done = false;
            break;
          }
          tc_fence_after();
          const float alpha = m_use > m_prev ? fast_exp2(m_prev - m_use) : 1.f;
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            uint32_t o[32];
            STA_TMEM_LD32(t_o + cc * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            STA_TMEM_ST32(t_o + cc * 32, o);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (lead) mbar_arrive(&p_full[b]);
          else mbar_arrive_remote(pf0 + b * 8);
        }
      }
      if (!done) break;
      // ---- item epilogue: merge the four partial sums of each row, normalise O
      const int ip = ii & 1;
      float* ls_i = lsum + ip * 512;
      float* ms_i = msum + ip * 256;
      ls_i[(grp * 2 + half) * 128 + r] = l_g;
      if (half == 0) ms_i[grp * 128 + r] = m_g;
      __syncwarp();
      if (lane == 0) mbar_arrive(sum_bar);
      if (!mbar_wait_warp(sum_bar, ii & 1, abort_flag) ||
          !mbar_wait_warp(o_full, ii & 1, abort_flag)) {
        done = false;
        break;
      }
      tc_fence_after();
      const float m0 = ms_i[r], m1 = ms_i[128 + r];
      const float mf = fmaxf(m0, m1);
      float l = 0.f;
      if (m0 != -INFINITY) l += (ls_i[r] + ls_i[128 + r]) * fast_exp2(m0 - mf);
      if (m1 != -INFINITY) l += (ls_i[256 + r] + ls_i[384 + r]) * fast_exp2(m1 - mf);
      const float inv = l > 0.f ? 1.f / l : 0.f;
      // this thread's 32 output columns
      const int c0 = grp * 64 + half * 32;
      uint32_t o[32];
      STA_TMEM_LD32(tmem + lane_off + C::kOCol + c0, o);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      // O may be overwritten by the next item's first P V from here on
      if (lane == 0) {
        if (lead) mbar_arrive(o_free);
        else mbar_arrive_remote(of0);
      }
      if (store) {
        int orow = qrow + r;
        if constexpr (R) orow = raster_row(p, orow);
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv, __uint_as_float(o[2 * e + 1]) * inv);
        uint4* dst = reinterpret_cast<uint4*>(p.out + static_cast<size_t>(orow) * C::D + c0);
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4)
          dst[v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
        if (p.lse != nullptr && grp == 0 && half == 0)
          p.lse[orow] = (mf + __log2f(l)) * 0.69314718055994531f;
      }
      gb += n;
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  cluster_sync();          // the peer no longer signals this CTA's barriers
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, C::kTmemCols);
  }
}

}  // namespace sta
