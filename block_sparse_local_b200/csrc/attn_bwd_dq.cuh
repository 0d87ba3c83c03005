// attn_bwd_dq.cuh - dQ of the STA backward pass for sm_100a.
//
// dQ = dS K / sqrt(d) with dS = P (dP - D), P = exp2(S log2(e)/sqrt(d) - LSE2),
// S = Q K^T and dP = dO V^T over the key blocks of the query block's window
// (the forward's tile lists).  One 128-row query block per CTA: Q and dO
// loaded once into shared memory and copied into TMEM, K and V streamed in
// separate TMA rings, K in three stages (released after dQ += dS K reads it)
// and V in two (released right after the dP MMA, its only reader).
//
// TMEM: the dQ accumulator in columns [0, 128); the resident Q and dO,
// packed bf16, in [128, 192) and [192, 256) (copied from shared memory by
// tcgen05.cp), so that S = Q K^T and dP = dO V^T are TS MMAs that read only
// K and V from shared memory (SS MMAs reading both operands there ran at two
// thirds of the tensor rate: shared-memory bandwidth); S(j) in [256, 384),
// dP(j) and then the packed dS(j) in [384, 512).  The elementwise warps copy
// S(j) into registers and release its columns at once, so S(j+1) is computed
// while they work on block j.  MMA order:
//   S(0) dP(0) S(1) | acc(0) dP(1) S(2) | acc(1) dP(2) S(3) | ...
// Warps: 0 TMA producer (one lane per operand panel), 1 MMA issuer (the whole
// warp waits, one elected lane issues; warp-uniform operands, constant
// accumulate flags), 2-17 elementwise: four warps per TMEM lane quarter, 32
// of the 128 key columns each (8 warps of 64 columns measured the same; 16
// need fewer registers per thread).
#pragma once

#include <type_traits>

#include "device_ptx.cuh"
#include "attn_bwd.cuh"

namespace sta {

constexpr int kDqEwWarps = 16;          // dQ kernel: elementwise warps
constexpr int kDqThreads = 64 + 32 * kDqEwWarps;

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

constexpr uint32_t kBwdDqColQ = 128;    // resident Q, packed bf16
constexpr uint32_t kBwdDqColDo = 192;   // resident dO, packed bf16
constexpr uint32_t kBwdDqColS = 256;    // S(j)
constexpr uint32_t kBwdDqColDp = 384;   // dP(j), then the packed dS(j)

// Descriptor offset (16-byte units) of k-step kk of a K-major block.
template <int D>
__device__ __forceinline__ uint32_t bwd_dq_kstep_off(int kk) {
  return static_cast<uint32_t>((kk >> 2) * BwdDqCfg<D>::kPanelBytes + (kk & 3) * 32) >> 4;
}

// Copy a resident block (K-major in shared memory) into TMEM as a packed
// bf16 A operand: k-step kk into columns [t + 8 kk, t + 8 kk + 8).
template <int D>
__device__ __forceinline__ void bwd_dq_copy_res(uint32_t t, uint64_t desc) {
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) tmem_cp_128x256b(t + kk * 8, desc + bwd_dq_kstep_off<D>(kk));
}

// D = A B^T over d (TS: A the resident block in TMEM, B a streamed K-major
// block in shared memory; 128 x 128).
template <int D>
__device__ __forceinline__ void bwd_dq_issue_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b) {
  constexpr uint32_t kIdS = idesc_bf16(128, 128, false);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk)
    umma_ts(d_tmem, a_tmem + kk * 8, b + bwd_dq_kstep_off<D>(kk), kIdS, kk > 0 ? 1u : 0u);
}

// dQ (+)= dS K: dS packed bf16 in TMEM (keys 32 g .. 32 g + 31 in columns
// [a + 32 g, a + 32 g + 16)), K an MN-major block (N = d).  ACC: accumulate
// flag of the first k-step.
template <int D, bool ACC>
__device__ __forceinline__ void bwd_dq_issue_acc(uint32_t d_tmem, uint32_t a_tmem, uint64_t b) {
  constexpr uint32_t kIdAcc = idesc_bf16(128, D, true);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint32_t acol = (kk >> 1) * 32 + (kk & 1) * 8;
    umma_ts(d_tmem, a_tmem + acol, b + ((kk * 16 * 128) >> 4), kIdAcc, (ACC || kk > 0) ? 1u : 0u);
  }
}

template <int D>
__global__ void __launch_bounds__(kDqThreads, 1)
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
  uint64_t* s_full = v_empty + VST;      // S(j) computed
  uint64_t* s_free = s_full + 1;         // every elementwise warp holds S(j): columns free
  uint64_t* dp_full = s_free + 1;        // dP(j) computed
  uint64_t* ds_full = dp_full + 1;       // packed dS(j) written
  uint64_t* acc_full = ds_full + 1;
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
    mbar_init(s_free, kDqEwWarps);
    mbar_init(dp_full, 1);
    mbar_init(ds_full, kDqEwWarps);
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
    // S(j+2) overwrites S's columns once every elementwise warp holds S(j+1)
    // in registers; dP(j+1) overwrites the packed dS(j) after acc(j), its
    // reader (tcgen05 ops of one thread execute in issue order).
    if (!skip) {
      const uint32_t tm = warp_uniform(tmem);
      const uint64_t d_q = sdesc_sw128(warp_uniform(smem_u32(smem + C::kQOff)), 16, 1024);
      const uint64_t d_do = sdesc_sw128(warp_uniform(smem_u32(smem + C::kDoOff)), 16, 1024);
      const uint64_t d_k = sdesc_sw128(warp_uniform(smem_u32(smem + C::kKOff)), 16, 1024);
      const uint64_t d_kmn =
          sdesc_sw128(warp_uniform(smem_u32(smem + C::kKOff)), C::kPanelBytes, 1024);
      const uint64_t d_v = sdesc_sw128(warp_uniform(smem_u32(smem + C::kVOff)), 16, 1024);
      auto issue_s = [&](int j) -> bool {      // S = Q K^T once K(j) has landed
        if (!mbar_wait_warp(&k_full[j % KST], (j / KST) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t off = (static_cast<uint32_t>(j % KST) * C::kBlockBytes) >> 4;
        if (elect_one()) {
          bwd_dq_issue_ts<D>(tm + kBwdDqColS, tm + kBwdDqColQ, d_k + off);
          umma_commit(s_full);
        }
        __syncwarp();
        return true;
      };
      auto issue_dp = [&](int j) -> bool {     // dP = dO V^T; V's only reader
        const int vs = j % VST;
        if (!mbar_wait_warp(&v_full[vs], (j / VST) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t off = (static_cast<uint32_t>(vs) * C::kBlockBytes) >> 4;
        if (elect_one()) {
          bwd_dq_issue_ts<D>(tm + kBwdDqColDp, tm + kBwdDqColDo, d_v + off);
          umma_commit(dp_full);
          umma_commit(&v_empty[vs]);
        }
        __syncwarp();
        return true;
      };
      bool ok = mbar_wait_warp(res_full, 0, abort_flag);
      if (ok) {
        tc_fence_after();
        if (elect_one()) {
          bwd_dq_copy_res<D>(tm + kBwdDqColQ, d_q);
          bwd_dq_copy_res<D>(tm + kBwdDqColDo, d_do);
        }
        __syncwarp();
        ok = issue_s(0) && issue_dp(0);
      }
      if (ok && n > 1) ok = mbar_wait_warp(s_free, 0, abort_flag) && issue_s(1);
      for (int j = 0; ok && j < n; ++j) {
        if (!mbar_wait_warp(ds_full, j & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t koff = (static_cast<uint32_t>(j % KST) * C::kBlockBytes) >> 4;
        if (elect_one()) {
          if (j > 0) bwd_dq_issue_acc<D, true>(tm, tm + kBwdDqColDp, d_kmn + koff);
          else bwd_dq_issue_acc<D, false>(tm, tm + kBwdDqColDp, d_kmn + koff);
          umma_commit(&k_empty[j % KST]);    // S(j) and acc(j) were K(j)'s readers
          if (j == n - 1) umma_commit(acc_full);
        }
        __syncwarp();
        if (j + 1 < n && !issue_dp(j + 1)) break;
        if (j + 2 < n && !(mbar_wait_warp(s_free, (j + 1) & 1, abort_flag) && issue_s(j + 2))) break;
      }
      if (elect_one()) umma_commit(mma_done);
      __syncwarp();
      mbar_wait_drain(mma_done, 0);
    }
  } else {
    // ------------------------------------------------------------ elementwise
    const int ks = warp - 2;
    const int cg = ks >> 2;                             // key columns [32 cg, 32 cg + 32)
    const int sub = warp & 3;                           // TMEM lane quarter
    const int r = sub * 32 + lane;                      // query row of the block
    const int my_row = item.q0 + r;
    if (!skip) {
      const uint32_t lane_off = static_cast<uint32_t>(sub * 32) << 16;
      const uint32_t t_s = tmem + lane_off + kBwdDqColS + cg * 32;
      const uint32_t t_dp = tmem + lane_off + kBwdDqColDp + cg * 32;
      const float2 sl2v = make_float2(p.scale_log2, p.scale_log2);
      const float row_nl2 = p.neg_lse2[my_row];         // -LSE in log2 units
      const float2 nl = make_float2(row_nl2, row_nl2);
      const float row_nd = p.neg_delta[my_row];         // -D
      const float2 nd = make_float2(row_nd, row_nd);
      bool done = true;
      for (int j = 0; j < n; ++j) {
        if (!mbar_wait_warp(s_full, j & 1, abort_flag)) { done = false; break; }
        tc_fence_after();
        uint32_t sr[32];
        STA_TMEM_LD32(t_s, sr);
        tmem_wait_ld();
        // S's columns may take the next block's S now
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free);
        // the text key block: keys >= text_len are padding
        int hi = 32;
        if (j >= nvid) hi = p.text_len - ((j - nvid) * 128 + cg * 32);
        // P = exp2(S sl2 - lse2), two columns at a time (packed f32x2 FMA; a
        // fixed share of the exponentials on the FMA pipe)
        float2 pr[16];
        auto exps = [&](auto with_mask) {
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int c = 2 * e;
            const float2 x = __ffma2_rn(
                make_float2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), sl2v, nl);
            float2 pe;
            if (exp2_on_fma(e)) {   // resolved at compile time (unrolled)
              pe = exp2_fma2(x);
            } else {
              pe = make_float2(fast_exp2(x.x), fast_exp2(x.y));
            }
            if constexpr (decltype(with_mask)::value) {
              if (c >= hi) pe.x = 0.f;
              if (c + 1 >= hi) pe.y = 0.f;
            }
            pr[e] = pe;
          }
        };
        if (hi < 32) {
          exps(std::true_type{});
        } else {
          exps(std::false_type{});
        }
        // dS = P (dP - D), packed to bf16 over the first 16 of this warp's own
        // 32 columns of dP(j)
        if (!mbar_wait_warp(dp_full, j & 1, abort_flag)) { done = false; break; }
        tc_fence_after();
        uint32_t dr[32], pk[16];
        STA_TMEM_LD32(t_dp, dr);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float2 ds = __fmul2_rn(
              pr[e], __fadd2_rn(make_float2(__uint_as_float(dr[2 * e]),
                                            __uint_as_float(dr[2 * e + 1])), nd));
          pk[e] = pack_bf16x2(ds.x, ds.y);
        }
        STA_TMEM_ST16(t_dp, pk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(ds_full);
      }
      if (done && mbar_wait_warp(acc_full, 0, abort_flag)) {
        tc_fence_after();
        // each warp writes D / 4 columns of its rows of dQ
        constexpr int kQCols = D / 4;
        const uint32_t t_acc = tmem + lane_off + cg * kQCols;
        uint4* dst = reinterpret_cast<uint4*>(p.out_a + static_cast<size_t>(my_row) * D +
                                              cg * kQCols);
#pragma unroll
        for (int cc = 0; cc < kQCols / 16; ++cc) {
          uint32_t o[16];
          STA_TMEM_LD16(t_acc + cc * 16, o);
          tmem_wait_ld();
          uint32_t pk2[8];
#pragma unroll
          for (int e = 0; e < 8; ++e)
            pk2[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * p.scale,
                                 __uint_as_float(o[2 * e + 1]) * p.scale);
          dst[cc * 2] = make_uint4(pk2[0], pk2[1], pk2[2], pk2[3]);
          dst[cc * 2 + 1] = make_uint4(pk2[4], pk2[5], pk2[6], pk2[7]);
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
