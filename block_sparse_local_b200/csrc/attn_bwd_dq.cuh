// attn_bwd_dq.cuh - dQ of the STA backward pass for sm_100a.
//
// dQ = dS K / sqrt(d) with dS = P (dP - D), P = exp2(S log2(e)/sqrt(d) - LSE2),
// S = Q K^T and dP = dO V^T over the key blocks of the query block's window
// (the forward's tile lists).  One 128-row query block per CTA: Q and dO
// resident in shared memory, K and V streamed in separate TMA rings, K in
// three stages (released after dQ += dS K reads it) and V in two (released
// right after the dP MMA, its only reader).
//
// TMEM: the dQ accumulator in columns [0, 128); S(j) of key block j alternates
// between [128, 256) and [384, 512); dP(j) in [256, 384).  The elementwise
// warps first copy S(j) and dP(j) into registers (after which [256, 384) may
// take dP(j+1)) and then write their packed bf16 dS(j) over their own columns
// of S(j), which dQ += dS K reads.  So the tensor cores compute S(j+1) and
// dP(j+1) while the elementwise warps work on block j, and the accumulate
// MMA of block j follows them.
// Warps: 0 TMA producer (one lane per operand panel), 1 MMA issuer (the whole
// warp waits, one elected lane issues; warp-uniform operands, constant
// accumulate flags), 2-9 elementwise: two warps per TMEM lane quarter, 64 of
// the 128 key columns each.
#pragma once

#include <type_traits>

#include "device_ptx.cuh"
#include "attn_bwd.cuh"

namespace sta {

template <int D>
struct BwdDqCfg {
  static constexpr int kPanels = D / 64;
  static constexpr int kPanelBytes = 128 * 128;
  static constexpr int kBlockBytes = 128 * D * 2;
  static constexpr int kKStages = 3;
  static constexpr int kVStages = 2;
  static constexpr int kQOff = 0;
  static constexpr int kDoOff = kQOff + kBlockBytes;
  static constexpr int kKOff = kDoOff + kBlockBytes;
  static constexpr int kVOff = kKOff + kKStages * kBlockBytes;
  static constexpr int kBarOff = kVOff + kVStages * kBlockBytes;
  static constexpr int kSmemBytes = kBarOff + 256 + 1024;   // + 1024-byte alignment
  static_assert(kSmemBytes <= 232448, "shared memory of one CTA");
};

// TMEM column of S(j); dP always at 256.
__device__ __forceinline__ uint32_t bwd_dq_s_col(int j) { return (j & 1) ? 384u : 128u; }
constexpr uint32_t kBwdDqDpCol = 256;

// D = A B^T over d (SS, both K-major, 128 x 128).  a, b: block descriptors
// (address field already offset).
template <int D>
__device__ __forceinline__ void bwd_dq_issue_ss(uint32_t d_tmem, uint64_t a, uint64_t b) {
  constexpr uint32_t kIdS = idesc_bf16(128, 128, false);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = ((kk >> 2) * BwdDqCfg<D>::kPanelBytes + (kk & 3) * 32) >> 4;
    umma_ss(d_tmem, a + off, b + off, kIdS, kk > 0 ? 1u : 0u);
  }
}

// dQ (+)= dS K: dS packed bf16 in TMEM (keys 0..63 in columns [a, a+32) of
// the first column group, keys 64..127 in [a+64, a+96) of the second), K an
// MN-major block (N = d).  ACC: accumulate flag of the first k-step.
template <int D, bool ACC>
__device__ __forceinline__ void bwd_dq_issue_acc(uint32_t d_tmem, uint32_t a_tmem, uint64_t b) {
  constexpr uint32_t kIdAcc = idesc_bf16(128, D, true);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint32_t acol = (kk >> 2) * 64 + (kk & 3) * 8;
    umma_ts(d_tmem, a_tmem + acol, b + ((kk * 16 * 128) >> 4), kIdAcc, (ACC || kk > 0) ? 1u : 0u);
  }
}

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmap_q,
                       const __grid_constant__ CUtensorMap tmap_k,
                       const __grid_constant__ CUtensorMap tmap_v,
                       const __grid_constant__ CUtensorMap tmap_do, const BwdParams p) {
  using C = BwdDqCfg<D>;
  constexpr int KST = C::kKStages;
  constexpr int VST = C::kVStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* res_full = bars;
  uint64_t* k_full = res_full + 1;       // [KST]
  uint64_t* k_empty = k_full + KST;      // [KST]
  uint64_t* v_full = k_empty + KST;      // [VST]
  uint64_t* v_empty = v_full + VST;      // [VST]
  uint64_t* s_full = v_empty + VST;      // S(j) and dP(j) computed
  uint64_t* d_free = s_full + 1;         // the elementwise warps have loaded S(j), dP(j)
  uint64_t* p_full = d_free + 1;         // [2 by block parity] dS(j) stored
  uint64_t* acc_full = p_full + 2;
  uint64_t* mma_done = acc_full + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const WorkItem item = p.items[blockIdx.x];
  // debug build: the item and its list lie inside the arrays they index
  const bool item_ok = dbg_ok(item.q0 >= 0 && item.q0 + 128 <= p.dbg_rows &&
                              item.kv_base >= 0 && item.kv_base < p.dbg_rows &&
                              item.list >= 0 && item.list < p.dbg_lists) &&
                       dbg_ok(p.counts[item.list] >= 0 && p.counts[item.list] <= p.max_k);
  // the query block's key blocks: video tiles of its list, then the text block
  const int cnt = item_ok ? p.counts[item.list] : 0;
  const int* ids = p.ids + static_cast<size_t>(item_ok ? item.list : 0) * p.max_k;
  const int nvid = (cnt - p.text_sentinel) * p.tile_blocks;
  const int n = item_ok ? nvid + (p.text_sentinel ? p.text_blocks : 0) : 0;
  auto key_row = [&](int j) {
    if (j < nvid) {
      const int t = j / p.tile_blocks;
      return item.kv_base + ids[t] * p.V + (j - t * p.tile_blocks) * 128;
    }
    return item.kv_base + p.L_v + (j - nvid) * 128;
  };

  if (threadIdx.x == 0) {
    mbar_init(res_full, 1);
    for (int i = 0; i < KST; ++i) { mbar_init(&k_full[i], 1); mbar_init(&k_empty[i], 1); }
    for (int i = 0; i < VST; ++i) { mbar_init(&v_full[i], 1); mbar_init(&v_empty[i], 1); }
    mbar_init(s_full, 1);
    mbar_init(d_free, 8);
    for (int i = 0; i < 2; ++i) mbar_init(&p_full[i], 8);
    mbar_init(acc_full, 1);
    mbar_init(mma_done, 1);
    *abort_flag = (error_raised() || n <= 0) ? 1 : 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmap_q);
    tma_prefetch_desc(&tmap_k);
    tma_prefetch_desc(&tmap_v);
    tma_prefetch_desc(&tmap_do);
  }
  if (warp == 1) tmem_alloc(tmem_holder, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const bool skip = *abort_flag != 0;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // One lane per operand panel (a thread's TMA loads complete one after
    // another): lanes 0 .. kPanels-1 load Q and then the K ring, lanes
    // kPanels .. 2 kPanels-1 load dO and then the V ring; the panel-0 lane
    // of each posts the expected bytes.
    constexpr int kPanels = C::kPanels;
    if (lane < 2 * kPanels && !skip) {
      const uint64_t pol = policy_evict_last();
      const bool is_v = lane >= kPanels;
      const int pn = lane % kPanels;
      if (lane == 0) mbar_arrive_expect_tx(res_full, 2 * C::kBlockBytes);
      tma_load_2d_hint(smem + (is_v ? C::kDoOff : C::kQOff) + pn * C::kPanelBytes,
                       is_v ? &tmap_do : &tmap_q, res_full, pn * 64, item.q0, pol);
      const int nst = is_v ? VST : KST;
      uint64_t* full = is_v ? v_full : k_full;
      uint64_t* empty = is_v ? v_empty : k_empty;
      uint8_t* base = smem + (is_v ? C::kVOff : C::kKOff);
      const CUtensorMap* map = is_v ? &tmap_v : &tmap_k;
      for (int j = 0; j < n; ++j) {
        const int st = j % nst;
        if (j >= nst && !mbar_wait(&empty[st], ((j / nst) - 1) & 1, abort_flag)) break;
        const int row = key_row(j);
        if (!dbg_ok(row >= 0 && row + 128 <= p.dbg_rows)) {
          *abort_flag = 1;
          break;
        }
        if (pn == 0) mbar_arrive_expect_tx(&full[st], C::kBlockBytes);
        tma_load_2d_hint(base + st * C::kBlockBytes + pn * C::kPanelBytes, map, &full[st],
                         pn * 64, row, pol);
      }
      __syncwarp((1u << (2 * kPanels)) - 1u);
      // Leave no copy in flight: wait for the last load of every stage.
      if (lane == 0) {
        mbar_wait_drain(res_full, 0);
        for (int st = 0; st < KST && st < n; ++st) {
          const int last = st + ((n - 1 - st) / KST) * KST;
          mbar_wait_drain(&k_full[st], (last / KST) & 1);
        }
        for (int st = 0; st < VST && st < n; ++st) {
          const int last = st + ((n - 1 - st) / VST) * VST;
          mbar_wait_drain(&v_full[st], (last / VST) & 1);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Per key block j: S(j+1) into the S column block that the accumulate
    // MMA of block j-1 read (issued before it; tcgen05 MMAs of one thread
    // execute in issue order), dP(j+1) once the elementwise warps have
    // loaded dP(j), then dQ += dS(j) K(j).
    if (!skip) {
      const uint32_t tm = warp_uniform(tmem);
      const uint64_t d_q = sdesc_sw128(warp_uniform(smem_u32(smem + C::kQOff)), 16, 1024);
      const uint64_t d_do = sdesc_sw128(warp_uniform(smem_u32(smem + C::kDoOff)), 16, 1024);
      const uint64_t d_k = sdesc_sw128(warp_uniform(smem_u32(smem + C::kKOff)), 16, 1024);
      const uint64_t d_kmn =
          sdesc_sw128(warp_uniform(smem_u32(smem + C::kKOff)), C::kPanelBytes, 1024);
      const uint64_t d_v = sdesc_sw128(warp_uniform(smem_u32(smem + C::kVOff)), 16, 1024);
      auto issue_s = [&](int j) {       // S = Q K^T
        const uint32_t off = (static_cast<uint32_t>(j % KST) * C::kBlockBytes) >> 4;
        if (elect_one()) bwd_dq_issue_ss<D>(tm + bwd_dq_s_col(j), d_q, d_k + off);
        __syncwarp();
      };
      auto issue_dp = [&](int j) {      // dP = dO V^T; V's stage is free once it is done
        const int vs = j % VST;
        const uint32_t off = (static_cast<uint32_t>(vs) * C::kBlockBytes) >> 4;
        if (elect_one()) {
          bwd_dq_issue_ss<D>(tm + kBwdDqDpCol, d_do, d_v + off);
          umma_commit(s_full);
          umma_commit(&v_empty[vs]);
        }
        __syncwarp();
      };
      bool ok = mbar_wait_warp(res_full, 0, abort_flag) &&
                mbar_wait_warp(&k_full[0], 0, abort_flag) &&
                mbar_wait_warp(&v_full[0], 0, abort_flag);
      if (ok) {
        tc_fence_after();
        issue_s(0);
        issue_dp(0);
      }
      for (int j = 0; ok && j < n; ++j) {
        const int jn = j + 1;
        const bool more = jn < n;
        if (more) {
          // K(j+1) and V(j+1) (both long loaded, as a rule) before S(j+1),
          // so only the wait for the elementwise warps sits between the two
          if (!mbar_wait_warp(&k_full[jn % KST], (jn / KST) & 1, abort_flag)) break;
          if (!mbar_wait_warp(&v_full[jn % VST], (jn / VST) & 1, abort_flag)) break;
          tc_fence_after();
          issue_s(jn);
          if (!mbar_wait_warp(d_free, j & 1, abort_flag)) break;
          tc_fence_after();
          issue_dp(jn);
        }
        if (!mbar_wait_warp(&p_full[j & 1], (j >> 1) & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t koff = (static_cast<uint32_t>(j % KST) * C::kBlockBytes) >> 4;
        if (elect_one()) {
          if (j > 0) bwd_dq_issue_acc<D, true>(tm, tm + bwd_dq_s_col(j), d_kmn + koff);
          else bwd_dq_issue_acc<D, false>(tm, tm + bwd_dq_s_col(j), d_kmn + koff);
          umma_commit(&k_empty[j % KST]);
          if (!more) umma_commit(acc_full);
        }
        __syncwarp();
      }
      if (elect_one()) umma_commit(mma_done);
      __syncwarp();
      mbar_wait_drain(mma_done, 0);
    }
  } else {
    // ------------------------------------------------------------ elementwise
    const int ks = warp - 2;
    const int half = ks >> 2;                           // key columns [64 half, 64 half + 64)
    const int sub = warp & 3;                           // TMEM lane quarter
    const int r = sub * 32 + lane;                      // query row of the block
    const int my_row = item.q0 + r;
    if (!skip) {
      const uint32_t lane_off = static_cast<uint32_t>(sub * 32) << 16;
      const float sl2 = p.scale_log2;
      const float row_nl2 = p.neg_lse2[my_row];         // -LSE in log2 units
      const float row_nd = p.neg_delta[my_row];         // -D
      bool done = true;
      for (int j = 0; j < n; ++j) {
        if (!mbar_wait_warp(s_full, j & 1, abort_flag)) { done = false; break; }
        tc_fence_after();
        const uint32_t t_s = tmem + lane_off + bwd_dq_s_col(j) + half * 64;
        const uint32_t t_dp = tmem + lane_off + kBwdDqDpCol + half * 64;
        uint32_t sr[64], dr[64];
        STA_TMEM_LD32(t_s, (sr + 0));
        STA_TMEM_LD32(t_s + 32, (sr + 32));
        STA_TMEM_LD32(t_dp, (dr + 0));
        STA_TMEM_LD32(t_dp + 32, (dr + 32));
        tmem_wait_ld();
        // dP's columns may take the next block's dP now
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(d_free);
        // the text key block: keys >= text_len are padding
        int hi = 64;
        if (j >= nvid) hi = p.text_len - ((j - nvid) * 128 + half * 64);
        uint32_t pk[32];
        // dS = P (dP - D), P = exp2(S sl2 - lse2), two columns at a time
        // (packed f32x2 FMA / ADD / MUL; a fixed share of the exponentials on
        // the FMA pipe), packed to bf16 as they come
        auto elementwise = [&](auto with_mask) {
          const float2 sl2v = make_float2(sl2, sl2);
          const float2 nl = make_float2(row_nl2, row_nl2);
          const float2 nd = make_float2(row_nd, row_nd);
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int c = 2 * e;
            const float2 x = __ffma2_rn(
                make_float2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), sl2v, nl);
            float2 pr;
            if (exp2_on_fma(e)) {   // resolved at compile time (unrolled)
              pr = exp2_fma2(x);
            } else {
              pr = make_float2(fast_exp2(x.x), fast_exp2(x.y));
            }
            if constexpr (decltype(with_mask)::value) {
              if (c >= hi) pr.x = 0.f;
              if (c + 1 >= hi) pr.y = 0.f;
            }
            const float2 ds = __fmul2_rn(
                pr, __fadd2_rn(make_float2(__uint_as_float(dr[c]), __uint_as_float(dr[c + 1])), nd));
            pk[e] = pack_bf16x2(ds.x, ds.y);
          }
        };
        if (hi < 64) {
          elementwise(std::true_type{});
        } else {
          elementwise(std::false_type{});
        }
        // packed dS over the first 32 of this warp's own 64 columns of S(j)
        STA_TMEM_ST32(t_s, pk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[j & 1]);
      }
      if (done && mbar_wait_warp(acc_full, 0, abort_flag)) {
        tc_fence_after();
        constexpr int kHalfCols = D / 2;
        const uint32_t t_acc = tmem + lane_off + half * kHalfCols;
        uint4* dst = reinterpret_cast<uint4*>(p.out_a + static_cast<size_t>(my_row) * D +
                                              half * kHalfCols);
#pragma unroll
        for (int cc = 0; cc < kHalfCols / 32; ++cc) {
          uint32_t o[32];
          STA_TMEM_LD32(t_acc + cc * 32, o);
          tmem_wait_ld();
          uint32_t pk2[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pk2[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * p.scale,
                                 __uint_as_float(o[2 * e + 1]) * p.scale);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            dst[cc * 4 + v4] = make_uint4(pk2[4 * v4], pk2[4 * v4 + 1], pk2[4 * v4 + 2],
                                          pk2[4 * v4 + 3]);
        }
      }
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace sta
