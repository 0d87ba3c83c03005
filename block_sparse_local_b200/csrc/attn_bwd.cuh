// attn_bwd.cuh - STA backward pass for sm_100a (dQ, dK, dV from the saved
// log-sum-exp of the forward).
//
// The STA pages give the forward only; the backward is the gradient of that
// function.  With S = Q K^T / sqrt(d) on allowed pairs, P = softmax(S),
// D_i = sum_c dO_ic O_ic:  dP = dO V^T,  dS = P (dP - D),
// dQ = dS K / sqrt(d),  dK = dS^T Q / sqrt(d),  dV = P^T dO.
//
// This file: the preprocessing (D and the log2-domain LSE), the transposed
// tile lists, and the dK/dV kernel, one 128-row key block per CTA: resident
// K, V; streams the query blocks whose windows hold that key tile
// (transposed tile lists), with their -LSE2 and -D.  TMEM: dV [0, d),
// dK [d, 2d).  The dQ kernel is in attn_bwd_dq.cuh.
// Each streamed 128-row block is worked on as two 64-row units, alternating
// between two TMEM score buffers at columns 256 and 384 (S or S^T in 64
// columns, dP or dP^T in the next 64), so the tensor cores compute the next
// unit's scores while the elementwise warps turn this unit's scores into P
// and dS: with one 128-row buffer (the accumulators leave room for no more
// at d = 128) the score MMAs, the elementwise work and the accumulate MMAs
// ran strictly one after another.
// Warps: 0 TMA producer (one lane per operand panel), 1 MMA issuer (S and dP
// by SS tcgen05.mma with N = 64, then the accumulators by TS tcgen05.mma with
// P / dS from TMEM, K = 64), 2-9 elementwise: two warps per TMEM lane
// quarter, 32 of the unit's 64 columns each.  A warp writes its packed bf16
// P / dS into the first 16 of its own 32 columns, so no warp overwrites
// scores another warp still has to read; the accumulate MMAs take the two
// column groups as two K ranges.
#pragma once

#include <type_traits>

#include "device_ptx.cuh"
#include "attn_fwd.cuh"

namespace sta {

constexpr int kBwdThreads = 320;

struct BwdParams {
  const WorkItem* items;
  const int* counts;      // lists (forward lists for dQ, transposed for dK/dV)
  const int* ids;
  int max_k;
  int tile_blocks;
  int V;
  int L_v;
  int text_len;
  int text_blocks;        // dQ: key blocks of the text block with valid keys
  int text_sentinel;      // lists end with the text block
  float scale_log2;       // log2(e) / sqrt(d)
  float scale;            // 1 / sqrt(d)
  const float* neg_lse2;  // [rows] minus the log-sum-exp in log2 units
  const float* neg_delta; // [rows] minus D
  __nv_bfloat16* out_a;   // dQ (dQ kernel) or dK (dK/dV kernel)
  __nv_bfloat16* out_b;   // dV (dK/dV kernel)
  int dbg_rows;           // rows of every [rows, d] tensor (debug-build bounds checks)
  int dbg_lists;          // rows of the lists
};

template <int D>
struct BwdCfg {
  static constexpr int kPanels = D / 64;
  static constexpr int kPanelBytes = 128 * 128;
  static constexpr int kBlockBytes = 128 * D * 2;
  static constexpr int kStages = 2;
  static constexpr int kResA = 0;                                  // K (dKV) / Q (dQ)
  static constexpr int kResB = kResA + kBlockBytes;                // V (dKV) / dO (dQ)
  static constexpr int kStream = kResB + kBlockBytes;              // per stage: 2 blocks + vec
  static constexpr int kStageBytes = 2 * kBlockBytes + 1024;
  static constexpr int kBarOff = kStream + kStages * kStageBytes;
  static constexpr int kSmemBytes = kBarOff + 256 + 1024;
};

// One warp per two rows: D[row] = sum_c dO[row,c] * O[row,c] (fp32) and the
// log-sum-exp converted to log2 units, both stored negated (the backward
// kernels add them: P = exp2(S log2(e)/sqrt(d) + neg_lse2), dP + neg_delta).
template <int D>
__global__ void __launch_bounds__(256) bwd_preprocess_kernel(
    const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dout,
    const float* __restrict__ lse, float* __restrict__ neg_delta,
    float* __restrict__ neg_lse2, long long rows) {
  constexpr int kLanes = D / 8;                       // 16-byte vectors per row
  constexpr int kRowsPerWarp = 32 / kLanes;
  const long long warp = (blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const long long row = warp * kRowsPerWarp + lane / kLanes;
  float acc = 0.f;
  if (row < rows) {
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(o + row * D) + lane % kLanes);
    const uint4 b = __ldg(reinterpret_cast<const uint4*>(dout + row * D) + lane % kLanes);
    const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 fa = __bfloat1622float2(pa[e]);
      const float2 fb = __bfloat1622float2(pb[e]);
      acc = fmaf(fa.x, fb.x, acc);
      acc = fmaf(fa.y, fb.y, acc);
    }
  }
#pragma unroll
  for (int off = kLanes / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (row < rows && lane % kLanes == 0) {
    neg_delta[row] = -acc;
    neg_lse2[row] = -lse[row] * 1.4426950408889634f;
  }
}

// Transposed tile lists: for key tile k of window class c, the ascending query
// tiles whose window box holds k, then the text query block NV when has_text
// (text queries see every video key).  Row NV (text keys, when has_text):
// every query tile, then NV.  One thread per (class, key row).
__global__ void __launch_bounds__(128) kv_tile_list_transposed_kernel(
    int* __restrict__ counts, int* __restrict__ ids, const ListWindows windows, int nclass,
    ListGeom g, int has_text) {
  const int gid = blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= nclass * g.NQ) return;
  const int cls = gid / g.NQ;
  const int row = gid - cls * g.NQ;
  int* out = ids + static_cast<size_t>(gid) * g.max_k;
  int n = 0;
  if (row < g.NV) {
    const int kw = row % g.NW, kh = (row / g.NW) % g.NH, kt = row / (g.NW * g.NH);
    for (int q = 0; q < g.NV; ++q) {
      const int qw = q % g.NW, qh = (q / g.NW) % g.NH, qt = q / (g.NW * g.NH);
      int s0, e0, s1, e1, s2, e2;
      window_range(qt, windows.w[cls * 3 + 0], g.NT, s0, e0);
      window_range(qh, windows.w[cls * 3 + 1], g.NH, s1, e1);
      window_range(qw, windows.w[cls * 3 + 2], g.NW, s2, e2);
      if (kt >= s0 && kt < s0 + e0 && kh >= s1 && kh < s1 + e1 && kw >= s2 && kw < s2 + e2)
        out[n++] = q;
    }
  } else {
    for (int q = 0; q < g.NV; ++q) out[n++] = q;
  }
  if (has_text) out[n++] = g.NV;
  counts[gid] = n;
  for (int i = n; i < g.max_k; ++i) out[i] = -1;
}

// TMEM columns: the accumulators (dV at 0 and dK at d, or dQ at 0), then two
// score buffers of one 64-row unit each: S (or S^T) in 64 columns, dP (or
// dP^T) in the next 64.
constexpr uint32_t kBwdBufCol = 256;

// Scores of one 64-row unit of a streamed block: D = A B^T over d (SS, both
// K-major, M = 128 resident rows, N = 64).  a: resident block descriptor, b:
// descriptor of the unit's first row (address field already offset).
template <int D>
__device__ __forceinline__ void bwd_issue_ss_unit(uint32_t d_tmem, uint64_t a, uint64_t b) {
  using C = BwdCfg<D>;
  constexpr uint32_t kIdS = idesc_bf16(128, 64, false);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = ((kk >> 2) * C::kPanelBytes + (kk & 3) * 32) >> 4;
    umma_ss(d_tmem, a + off, b + off, kIdS, kk > 0 ? 1u : 0u);
  }
}

// acc (+)= A B over one 64-row unit: A packed bf16 in TMEM, K = 64 rows of
// the unit, columns [a, a+16) (rows 0..31, first column group) and
// [a+32, a+48) (rows 32..63, second group); B the unit's rows of a streamed
// block as an MN-major operand (N = d).  ACC: accumulate flag of the first
// k-step.
template <int D, bool ACC>
__device__ __forceinline__ void bwd_issue_ts_unit(uint32_t d_tmem, uint32_t a_tmem, uint64_t b) {
  constexpr uint32_t kIdAcc = idesc_bf16(128, D, true);
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    const uint32_t acol = (kk >> 1) * 32 + (kk & 1) * 8;
    umma_ts(d_tmem, a_tmem + acol, b + ((kk * 16 * 128) >> 4), kIdAcc, (ACC || kk > 0) ? 1u : 0u);
  }
}

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_dkv_kernel(const __grid_constant__ CUtensorMap tmap_q,
                    const __grid_constant__ CUtensorMap tmap_k,
                    const __grid_constant__ CUtensorMap tmap_v,
                    const __grid_constant__ CUtensorMap tmap_do, const BwdParams p) {
  using C = BwdCfg<D>;
  constexpr int ST = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* res_full = bars;
  uint64_t* full = res_full + 1;         // [ST]
  uint64_t* empty = full + ST;           // [ST]
  uint64_t* s_full = empty + ST;         // [2] per score buffer
  uint64_t* p_full = s_full + 2;         // [2]
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
  // stream: key blocks of the query block (dQ) or query blocks of the key block (dK/dV)
  const int cnt = item_ok ? p.counts[item.list] : 0;
  const int* ids = p.ids + static_cast<size_t>(item_ok ? item.list : 0) * p.max_k;
  const int nvid = (cnt - p.text_sentinel) * p.tile_blocks;
  const int n = item_ok ? nvid + (p.text_sentinel ? p.text_blocks : 0) : 0;
  auto stream_row = [&](int j) {
    if (j < nvid) {
      const int t = j / p.tile_blocks;
      return item.kv_base + ids[t] * p.V + (j - t * p.tile_blocks) * 128;
    }
    return item.kv_base + p.L_v + (j - nvid) * 128;
  };

  if (threadIdx.x == 0) {
    mbar_init(res_full, 1);
    for (int i = 0; i < ST; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 8);
    }
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
  const uint32_t s_res_a = smem_u32(smem + C::kResA);
  const uint32_t s_res_b = smem_u32(smem + C::kResB);
  const uint32_t s_stream = smem_u32(smem + C::kStream);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // A thread's TMA loads complete one after another, so every operand
    // panel has its own lane: lanes 0 .. kPanels-1 the panels of the first
    // streamed operand (Q for dK/dV, K for dQ) and of the resident K / Q,
    // lanes kPanels .. 2 kPanels-1 those of the second (dO / V, resident
    // V / dO), lane 2 kPanels the two 512-byte LSE / D copies (dK/dV).  Lane
    // 0 posts the expected bytes of every stage.
    constexpr int kPanels = C::kPanels;
    constexpr int kLanes = 2 * kPanels + 1;
    if (lane < kLanes && !skip) {
      const uint64_t pol = policy_evict_last();
      const int row0 = item.q0;   // the resident block
      const bool is_b = lane >= kPanels && lane < 2 * kPanels;
      const bool is_vec = lane == 2 * kPanels;
      const int pn = lane % kPanels;
      if (lane == 0) mbar_arrive_expect_tx(res_full, 2 * C::kBlockBytes);
      if (!is_vec) {
        const CUtensorMap* mres = is_b ? &tmap_v : &tmap_k;
        tma_load_2d_hint(smem + (is_b ? C::kResB : C::kResA) + pn * C::kPanelBytes, mres,
                         res_full, pn * 64, row0, pol);
      }
      const CUtensorMap* mstr = is_b ? &tmap_do : &tmap_q;
      for (int j = 0; j < n; ++j) {
        const int st = j % ST;
        if (j >= ST && !mbar_wait(&empty[st], ((j / ST) - 1) & 1, abort_flag)) break;
        const int row = stream_row(j);
        if (!dbg_ok(row >= 0 && row + 128 <= p.dbg_rows)) {
          *abort_flag = 1;
          break;
        }
        uint8_t* base = smem + C::kStream + st * C::kStageBytes;
        if (lane == 0) mbar_arrive_expect_tx(&full[st], 2 * C::kBlockBytes + 1024);
        if (!is_vec) {
          tma_load_2d_hint(base + (is_b ? C::kBlockBytes : 0) + pn * C::kPanelBytes, mstr,
                           &full[st], pn * 64, row, pol);
        } else {
          // the streamed query block's -lse2 and -D (2 x 512 bytes)
          asm volatile(
              "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], "
              "512, [%2];" ::"r"(smem_u32(base + 2 * C::kBlockBytes)),
              "l"(reinterpret_cast<uint64_t>(p.neg_lse2 + row)), "r"(smem_u32(&full[st]))
              : "memory");
          asm volatile(
              "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], "
              "512, [%2];" ::"r"(smem_u32(base + 2 * C::kBlockBytes + 512)),
              "l"(reinterpret_cast<uint64_t>(p.neg_delta + row)), "r"(smem_u32(&full[st]))
              : "memory");
        }
      }
      __syncwarp((1u << kLanes) - 1u);
      // Leave no copy in flight: wait for the last load of every stage.
      if (lane == 0) {
        mbar_wait_drain(res_full, 0);
        for (int st = 0; st < ST && st < n; ++st) {
          const int last = st + ((n - 1 - st) / ST) * ST;
          mbar_wait_drain(&full[st], (last / ST) & 1);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Whole warp waits, one elected lane (always the same) issues; every MMA
    // operand is warp-uniform and every accumulate flag a constant.
    if (!skip) {
      const uint32_t tm = warp_uniform(tmem);
      const uint64_t d_res_a = sdesc_sw128(warp_uniform(s_res_a), 16, 1024);
      const uint64_t d_res_b = sdesc_sw128(warp_uniform(s_res_b), 16, 1024);
      const uint64_t d_str_k = sdesc_sw128(warp_uniform(s_stream), 16, 1024);
      const uint64_t d_str_mn = sdesc_sw128(warp_uniform(s_stream), C::kPanelBytes, 1024);
      // Units u = 0 .. 2n-1: the two 64-row halves of streamed block u / 2,
      // in score buffer u % 2.  Scores of unit u + 2 go into the buffer that
      // the accumulate MMAs of unit u read, issued right after them (tcgen05
      // MMAs of one thread execute in issue order), so the scores of the next
      // unit are computed while the elementwise warps work on this one.
      const int U = 2 * n;
      auto issue_scores = [&](int u) {
        const int st = (u >> 1) % ST;
        const uint32_t so = (static_cast<uint32_t>(st) * C::kStageBytes + (u & 1) * 64 * 128) >> 4;
        const uint32_t sb = so + (C::kBlockBytes >> 4);
        const uint32_t buf = tm + kBwdBufCol + (u & 1) * 128;
        if (elect_one()) {
          bwd_issue_ss_unit<D>(buf, d_res_a, d_str_k + so);        // S^T = K Q^T  |  S = Q K^T
          bwd_issue_ss_unit<D>(buf + 64, d_res_b, d_str_k + sb);   // dP^T = V dO^T |  dP = dO V^T
          umma_commit(&s_full[u & 1]);
        }
        __syncwarp();
      };
      bool ok = mbar_wait_warp(res_full, 0, abort_flag) && mbar_wait_warp(&full[0], 0, abort_flag);
      if (ok) {
        tc_fence_after();
        issue_scores(0);
        issue_scores(1);
      }
      for (int u = 0; ok && u < U; ++u) {
        const int st = (u >> 1) % ST;
        if (!mbar_wait_warp(&p_full[u & 1], (u >> 1) & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t so = (static_cast<uint32_t>(st) * C::kStageBytes + (u & 1) * 64 * 128) >> 4;
        const uint32_t sb = so + (C::kBlockBytes >> 4);
        const uint32_t buf = tm + kBwdBufCol + (u & 1) * 128;
        if (elect_one()) {
          if (u > 0) {
            bwd_issue_ts_unit<D, true>(tm, buf, d_str_mn + sb);           // dV += P^T dO
            bwd_issue_ts_unit<D, true>(tm + D, buf + 64, d_str_mn + so);  // dK += dS^T Q
          } else {
            bwd_issue_ts_unit<D, false>(tm, buf, d_str_mn + sb);
            bwd_issue_ts_unit<D, false>(tm + D, buf + 64, d_str_mn + so);
          }
          if (u & 1) umma_commit(&empty[st]);   // both units of the stage consumed
          if (u == U - 1) umma_commit(acc_full);
        }
        __syncwarp();
        const int un = u + 2;
        if (un < U) {
          if ((un & 1) == 0) {
            const int jn = un >> 1;
            if (!mbar_wait_warp(&full[jn % ST], (jn / ST) & 1, abort_flag)) break;
            tc_fence_after();
          }
          issue_scores(un);
        }
      }
      if (elect_one()) umma_commit(mma_done);
      __syncwarp();
      mbar_wait_drain(mma_done, 0);
    }
  } else {
    // ------------------------------------------------------------ elementwise
    const int ks = warp - 2;
    const int half = ks >> 2;
    const int sub = warp & 3;
    const int r = sub * 32 + lane;                      // row of the resident block
    const int my_row = item.q0 + r;
    if (!skip) {
      const uint32_t lane_off = static_cast<uint32_t>(sub * 32) << 16;
      const float sl2 = p.scale_log2;
      // whether this key row is valid (padded text keys are not)
      bool row_valid = true;
      {
        const int off = my_row - item.kv_base;
        if (off >= p.L_v) row_valid = (off - p.L_v) < p.text_len;
      }
      bool done = true;
      for (int u = 0; u < 2 * n; ++u) {
        const int j = u >> 1;           // streamed block
        const int hu = u & 1;           // its 64-row half, and the score buffer
        const int st = j % ST;
        if (!mbar_wait_warp(&s_full[hu], j & 1, abort_flag)) { done = false; break; }
        if (!mbar_wait_warp(&full[st], (j / ST) & 1, abort_flag)) { done = false; break; }
        tc_fence_after();
        const uint32_t t_s = tmem + lane_off + kBwdBufCol + hu * 128 + half * 32;
        const uint32_t t_dp = t_s + 64;
        uint32_t sr[32], dr[32];
        STA_TMEM_LD32(t_s, sr);
        STA_TMEM_LD32(t_dp, dr);
        tmem_wait_ld();
        // padded text key rows give zero P and dS
        const bool masked = !__all_sync(0xffffffffu, row_valid);
        // -lse2 and -D of this warp's 32 streamed rows, 16-byte aligned in
        // the stage
        const float4* nl4p = reinterpret_cast<const float4*>(
            smem + C::kStream + st * C::kStageBytes + 2 * C::kBlockBytes) + hu * 16 + half * 8;
        const float4* nd4p = nl4p + 32;
        uint32_t pk_p[16], pk_ds[16];
        // P = exp2(S sl2 - lse2) and dS = P (dP - D), two columns at a time
        // (packed f32x2 FMA / ADD / MUL; a fixed share of the exponentials on
        // the FMA pipe), packed to bf16 as they come
        auto elementwise = [&](auto with_mask) {
          const float2 sl2v = make_float2(sl2, sl2);
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4) {
            const float4 nl4 = nl4p[e4];
            const float4 nd4 = nd4p[e4];
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
              const int e = 2 * e4 + h2;       // column pair
              const int c = 2 * e;
              const float2 nl = h2 ? make_float2(nl4.z, nl4.w) : make_float2(nl4.x, nl4.y);
              const float2 nd = h2 ? make_float2(nd4.z, nd4.w) : make_float2(nd4.x, nd4.y);
              const float2 x = __ffma2_rn(
                  make_float2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), sl2v, nl);
              float2 pr;
              if (exp2_on_fma(e)) {   // resolved at compile time (unrolled)
                pr = exp2_fma2(x);
              } else {
                pr = make_float2(fast_exp2(x.x), fast_exp2(x.y));
              }
              if constexpr (decltype(with_mask)::value) {
                if (!row_valid) pr = make_float2(0.f, 0.f);
              }
              const float2 ds = __fmul2_rn(
                  pr, __fadd2_rn(make_float2(__uint_as_float(dr[c]), __uint_as_float(dr[c + 1])),
                                 nd));
              pk_p[e] = pack_bf16x2(pr.x, pr.y);
              pk_ds[e] = pack_bf16x2(ds.x, ds.y);
            }
          }
        };
        if (masked) {
          elementwise(std::true_type{});
        } else {
          elementwise(std::false_type{});
        }
        // packed bf16 over the first 16 of this warp's own 32 columns, so no
        // warp overwrites scores another warp still has to read
        STA_TMEM_ST16(t_s, pk_p);     // P^T
        STA_TMEM_ST16(t_dp, pk_ds);   // dS^T
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[hu]);
      }
      if (done && mbar_wait_warp(acc_full, 0, abort_flag)) {
        tc_fence_after();
        constexpr int kHalfCols = D / 2;
        for (int a = 0; a < 2; ++a) {
          // a = 0 -> dV (unscaled), a = 1 -> dK (scaled)
          const uint32_t t_acc = tmem + lane_off + (a == 1 ? D : 0) + half * kHalfCols;
          const float sc = a == 0 ? 1.f : p.scale;
          __nv_bfloat16* dstp = a == 0 ? p.out_b : p.out_a;
          uint4* dst = reinterpret_cast<uint4*>(dstp + static_cast<size_t>(my_row) * D +
                                                half * kHalfCols);
#pragma unroll
          for (int cc = 0; cc < kHalfCols / 32; ++cc) {
            uint32_t o[32];
            STA_TMEM_LD32(t_acc + cc * 32, o);
            tmem_wait_ld();
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e)
              pk[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * sc, __uint_as_float(o[2 * e + 1]) * sc);
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4)
              dst[cc * 4 + v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2],
                                            pk[4 * v4 + 3]);
          }
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
