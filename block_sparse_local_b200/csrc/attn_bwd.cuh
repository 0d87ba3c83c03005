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
// (transposed tile lists), each pipeline stage holding one Q block, its dO
// block and its -D.  The dQ kernel is in attn_bwd_dq.cuh.
// Every MMA has N = 128 (the whole streamed block): an MMA with N = 64
// costs the tensor cores as long as one with N = 128, so 64-row units would
// cap the kernel at about three quarters of the tensor rate.  TMEM: dV and dK
// (fp32), chunk A = S^T of the streamed block, then its packed P^T, chunk B =
// dP^T, then the packed dS^T.  MMA order:
//   S(0) dP(0) | dV(0) S(1) dK(0) dP(1) | dV(1) S(2) dK(1) dP(2) | ...
// so the elementwise warps turn S(j) into P(j) while the tensor cores run
// dK(j-1) and dP(j), and dP(j) into dS(j) while they run dV(j) and S(j+1).
// The per-column -LSE2 of the exponentials is loaded from global memory (L1)
// before the wait for S(j), so its latency is off that phase's path; with
// 16-byte broadcast loads from shared memory it sat on it, behind the score
// MMAs' operand reads (measured: 46.6 vs 48.7 ms for the whole backward).
// Warps: 0 TMA producer (one lane per operand panel), 1 MMA issuer (scores
// by SS tcgen05.mma, the accumulators by TS tcgen05.mma with P^T / dS^T from
// TMEM), 2-17 elementwise: four warps per TMEM lane quarter, 32 of the 128
// streamed rows (score columns) each.  A warp writes its packed bf16 P^T /
// dS^T into the first 16 of its own 32 columns, so no warp overwrites scores
// another warp still has to read; the accumulate MMAs take two K steps of 16
// rows from each warp's packed columns.
#pragma once

#include <type_traits>

#include "device_ptx.cuh"
#include "attn_fwd.cuh"

namespace sta {

constexpr int kDkvEwWarps = 16;         // dK/dV kernel: elementwise warps
constexpr int kDkvThreads = 64 + 32 * kDkvEwWarps;
// Exponentials of the dK/dV kernel on the FMA pipe: this many of every 8
// column pairs (the rest on the ex2 unit).
#ifndef STA_DKV_EXP2_FMA_PAIRS
#define STA_DKV_EXP2_FMA_PAIRS 2
#endif
constexpr int kDkvExp2FmaPairs = STA_DKV_EXP2_FMA_PAIRS;

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
  static constexpr int kResA = 0;                                  // resident K
  static constexpr int kResB = kResA + kBlockBytes;                // resident V
  static constexpr int kStream = kResB + kBlockBytes;              // per stage: Q, dO, -D
  // -D takes 512 bytes; the stage stride stays a multiple of 1024 so that
  // every 128-byte-swizzled block starts on a 1024-byte boundary
  static constexpr int kStageBytes = 2 * kBlockBytes + 1024;
  static constexpr int kBarOff = kStream + kStages * kStageBytes;
  static constexpr int kSmemBytes = kBarOff + 256 + 1024;   // + 1024-byte alignment
  static_assert(kSmemBytes <= 232448, "shared memory of one CTA");
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

// TMEM columns of the two 128-column chunks (the accumulators: dV at 0, dK
// at d).
constexpr uint32_t kDkvColA = 256;
constexpr uint32_t kDkvColB = 384;

// Scores of a streamed block: D = A B^T over d (SS, both K-major, M = 128
// resident rows, N = 128 streamed rows).  a: resident block descriptor, b:
// descriptor of the streamed block (address field already offset).
template <int D>
__device__ __forceinline__ void bwd_issue_scores(uint32_t d_tmem, uint64_t a, uint64_t b) {
  using C = BwdCfg<D>;
  constexpr uint32_t kIdS = idesc_bf16(128, 128, false);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = ((kk >> 2) * C::kPanelBytes + (kk & 3) * 32) >> 4;
    umma_ss(d_tmem, a + off, b + off, kIdS, kk > 0 ? 1u : 0u);
  }
}

// acc (+)= A B over a streamed block: A packed bf16 in TMEM, K = the 128
// streamed rows in four groups of 32 (rows 32 g .. 32 g + 31 packed into
// columns [a + 32 g, a + 32 g + 16)); B the streamed block as an MN-major
// operand (N = d).  ACC: accumulate flag of the first k-step.
template <int D, bool ACC>
__device__ __forceinline__ void bwd_issue_acc(uint32_t d_tmem, uint32_t a_tmem, uint64_t b) {
  constexpr uint32_t kIdAcc = idesc_bf16(128, D, true);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint32_t acol = (kk >> 1) * 32 + (kk & 1) * 8;
    umma_ts(d_tmem, a_tmem + acol, b + ((kk * 16 * 128) >> 4), kIdAcc, (ACC || kk > 0) ? 1u : 0u);
  }
}

template <int D>
__global__ void __launch_bounds__(kDkvThreads, 1)
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
  uint64_t* s_full = empty + ST;         // S^T of the current block in chunk A
  uint64_t* dp_full = s_full + 1;        // dP^T in chunk B
  uint64_t* p_full = dp_full + 1;        // packed P^T written (every elementwise warp)
  uint64_t* ds_full = p_full + 1;        // packed dS^T written
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
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(p_full, kDkvEwWarps);
    mbar_init(ds_full, kDkvEwWarps);
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
    // panel has its own lane: lanes 0 .. kPanels-1 the panels of resident K
    // and of the streamed Q blocks, lanes kPanels .. 2 kPanels-1 those of
    // resident V and of the streamed dO blocks, lane 2 kPanels the 512-byte
    // -D copies.  Lane 0 posts the expected bytes of every stage.
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
        if (lane == 0) mbar_arrive_expect_tx(&full[st], 2 * C::kBlockBytes + 512);
        if (!is_vec) {
          tma_load_2d_hint(base + (is_b ? C::kBlockBytes : 0) + pn * C::kPanelBytes, mstr,
                           &full[st], pn * 64, row, pol);
        } else {
          // the streamed query block's -D (512 bytes)
          asm volatile(
              "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], "
              "512, [%2];" ::"r"(smem_u32(base + 2 * C::kBlockBytes)),
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
    // operand is warp-uniform and every accumulate flag a constant.  S(j+1)
    // overwrites chunk A after dV(j), the last reader of P(j), and dP(j+1)
    // chunk B after dK(j), the last reader of dS(j): tcgen05 MMAs of one
    // thread execute in issue order.
    if (!skip) {
      const uint32_t tm = warp_uniform(tmem);
      const uint64_t d_res_a = sdesc_sw128(warp_uniform(s_res_a), 16, 1024);
      const uint64_t d_res_b = sdesc_sw128(warp_uniform(s_res_b), 16, 1024);
      const uint64_t d_str_k = sdesc_sw128(warp_uniform(s_stream), 16, 1024);
      const uint64_t d_str_mn = sdesc_sw128(warp_uniform(s_stream), C::kPanelBytes, 1024);
      // descriptor offsets of a stage's first streamed block (Q or K) and of
      // its second (dO or V)
      auto stage_off = [](int j) {
        return static_cast<uint32_t>((j % ST) * C::kStageBytes) >> 4;
      };
      constexpr uint32_t kSecond = C::kBlockBytes >> 4;
      bool ok = mbar_wait_warp(res_full, 0, abort_flag) && mbar_wait_warp(&full[0], 0, abort_flag);
      if (ok) {
        tc_fence_after();
        if (elect_one()) {
          bwd_issue_scores<D>(tm + kDkvColA, d_res_a, d_str_k);              // S^T = K Q^T
          umma_commit(s_full);
          bwd_issue_scores<D>(tm + kDkvColB, d_res_b, d_str_k + kSecond);    // dP^T = V dO^T
          umma_commit(dp_full);
        }
        __syncwarp();
      }
      for (int j = 0; ok && j < n; ++j) {
        const uint32_t so = stage_off(j);
        const bool more = j + 1 < n;
        if (!mbar_wait_warp(p_full, j & 1, abort_flag)) break;
        tc_fence_after();
        if (elect_one()) {
          if (j > 0) {
            bwd_issue_acc<D, true>(tm, tm + kDkvColA, d_str_mn + so + kSecond);    // dV += P^T dO
          } else {
            bwd_issue_acc<D, false>(tm, tm + kDkvColA, d_str_mn + so + kSecond);
          }
        }
        __syncwarp();
        if (more) {
          const int jn = j + 1;
          if (!mbar_wait_warp(&full[jn % ST], (jn / ST) & 1, abort_flag)) break;
          tc_fence_after();
          if (elect_one()) {
            bwd_issue_scores<D>(tm + kDkvColA, d_res_a, d_str_k + stage_off(jn));
            umma_commit(s_full);
          }
          __syncwarp();
        }
        if (!mbar_wait_warp(ds_full, j & 1, abort_flag)) break;
        tc_fence_after();
        if (elect_one()) {
          if (j > 0) {
            bwd_issue_acc<D, true>(tm + D, tm + kDkvColB, d_str_mn + so);           // dK += dS^T Q
          } else {
            bwd_issue_acc<D, false>(tm + D, tm + kDkvColB, d_str_mn + so);
          }
          umma_commit(&empty[j % ST]);   // every reader of the stage has been issued
          if (more) {
            bwd_issue_scores<D>(tm + kDkvColB, d_res_b, d_str_k + stage_off(j + 1) + kSecond);
            umma_commit(dp_full);
          } else {
            umma_commit(acc_full);
          }
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
    const int cg = ks >> 2;                             // 32-column group of the scores
    const int sub = warp & 3;                           // TMEM lane quarter
    const int r = sub * 32 + lane;                      // row of the resident block
    const int my_row = item.q0 + r;
    if (!skip) {
      const uint32_t lane_off = static_cast<uint32_t>(sub * 32) << 16;
      const uint32_t t_a = tmem + lane_off + kDkvColA + cg * 32;
      const uint32_t t_b = tmem + lane_off + kDkvColB + cg * 32;
      const float2 sl2v = make_float2(p.scale_log2, p.scale_log2);
      // whether this key row is valid (padded text keys are not)
      bool row_valid = true;
      {
        const int off = my_row - item.kv_base;
        if (off >= p.L_v) row_valid = (off - p.L_v) < p.text_len;
      }
      // padded text key rows give zero P and dS
      const bool masked = !__all_sync(0xffffffffu, row_valid);
      bool done = true;
      for (int j = 0; j < n; ++j) {
        const int st = j % ST;
        // -lse2 of this warp's 32 streamed rows from global memory (the same
        // address in every lane), loaded before the wait for S(j)
        float4 nl4v[8];
        {
          const float4* g = reinterpret_cast<const float4*>(p.neg_lse2 + stream_row(j) + cg * 32);
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4) nl4v[e4] = __ldg(g + e4);
        }
        if (!mbar_wait_warp(s_full, j & 1, abort_flag)) { done = false; break; }
        if (!mbar_wait_warp(&full[st], (j / ST) & 1, abort_flag)) { done = false; break; }
        tc_fence_after();
        // -D of this warp's 32 streamed rows, 16-byte aligned in the stage
        const float4* nd4p = reinterpret_cast<const float4*>(
            smem + C::kStream + st * C::kStageBytes + 2 * C::kBlockBytes) + cg * 8;
        // P = exp2(S sl2 - lse2), two columns at a time (packed f32x2 FMA; a
        // fixed share of the exponentials on the FMA pipe); kept in fp32 for
        // dS and packed to bf16 as P^T over the first 16 of the warp's columns
        float2 pr[16];
        {
          uint32_t sr[32], pk[16];
          STA_TMEM_LD32(t_a, sr);
          tmem_wait_ld();
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4) {
            const float4 nl4 = nl4v[e4];
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
              const int e = 2 * e4 + h2;       // column pair
              const float2 nl = h2 ? make_float2(nl4.z, nl4.w) : make_float2(nl4.x, nl4.y);
              const float2 x = __ffma2_rn(
                  make_float2(__uint_as_float(sr[2 * e]), __uint_as_float(sr[2 * e + 1])), sl2v, nl);
              float2 pe;
              if (exp2_on_fma_of<kDkvExp2FmaPairs>(e)) {   // resolved at compile time
                pe = exp2_fma2(x);
              } else {
                pe = make_float2(fast_exp2(x.x), fast_exp2(x.y));
              }
              if (masked && !row_valid) pe = make_float2(0.f, 0.f);
              pr[e] = pe;
              pk[e] = pack_bf16x2(pe.x, pe.y);
            }
          }
          STA_TMEM_ST16(t_a, pk);     // P^T
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full);
        // dS = P (dP - D)
        if (!mbar_wait_warp(dp_full, j & 1, abort_flag)) { done = false; break; }
        tc_fence_after();
        {
          uint32_t dr[32], pk[16];
          STA_TMEM_LD32(t_b, dr);
          tmem_wait_ld();
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4) {
            const float4 nd4 = nd4p[e4];
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
              const int e = 2 * e4 + h2;
              const float2 nd = h2 ? make_float2(nd4.z, nd4.w) : make_float2(nd4.x, nd4.y);
              const float2 ds = __fmul2_rn(
                  pr[e], __fadd2_rn(make_float2(__uint_as_float(dr[2 * e]),
                                                __uint_as_float(dr[2 * e + 1])), nd));
              pk[e] = pack_bf16x2(ds.x, ds.y);
            }
          }
          STA_TMEM_ST16(t_b, pk);     // dS^T
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(ds_full);
      }
      if (done && mbar_wait_warp(acc_full, 0, abort_flag)) {
        tc_fence_after();
        // each warp writes D / 4 columns of its rows of dV and of dK
        constexpr int kQCols = D / 4;
        for (int a = 0; a < 2; ++a) {
          // a = 0 -> dV (unscaled), a = 1 -> dK (scaled)
          const uint32_t t_acc = tmem + lane_off + (a == 1 ? D : 0) + cg * kQCols;
          const float sc = a == 0 ? 1.f : p.scale;
          __nv_bfloat16* dstp = a == 0 ? p.out_b : p.out_a;
          uint4* dst = reinterpret_cast<uint4*>(dstp + static_cast<size_t>(my_row) * D +
                                                cg * kQCols);
#pragma unroll
          for (int cc = 0; cc < kQCols / 16; ++cc) {
            uint32_t o[16];
            STA_TMEM_LD16(t_acc + cc * 16, o);
            tmem_wait_ld();
            uint32_t pk[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
              pk[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * sc, __uint_as_float(o[2 * e + 1]) * sc);
            dst[cc * 2] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            dst[cc * 2 + 1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
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
