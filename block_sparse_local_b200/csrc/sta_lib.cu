// sta_lib.cu - host side of libsta.so: argument checks, planning, TMA
// descriptors, workspace and launches behind the C ABI of include/sta.h.
//
// One translation unit: the kernels are included from the .cuh files so the
// device error word has a single definition.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <queue>
#include <string>
#include <vector>

#include "sta.h"
#include "device_ptx.cuh"
#include "reorder.cuh"
#include "tile_lists.cuh"
#include "attn_fwd.cuh"
#include "attn_fwd_pair.cuh"
#include "hilbert.cuh"
#include "attn_bwd.cuh"
#include "attn_bwd_dq.cuh"

namespace {

using sta::FwdParams;
using sta::Mode;
using sta::WorkItem;

constexpr int kMaxClasses = sta::kMaxWindowClasses;

#define STA_CUDA_TRY(expr)                         \
  do {                                             \
    cudaError_t e_ = (expr);                       \
    if (e_ != cudaSuccess) return STA_ERR_CUDA;    \
  } while (0)

// ------------------------------------------------------------------ device
struct DeviceInfo {
  bool checked = false;
  bool sm100 = false;
  int num_sms = 0;
};

std::mutex g_mu;
DeviceInfo g_dev[64];

sta_status current_device(int* dev) {
  if (cudaGetDevice(dev) != cudaSuccess || *dev < 0 || *dev >= 64) return STA_ERR_CUDA;
  DeviceInfo& di = g_dev[*dev];
  if (!di.checked) {
    int major = 0, minor = 0, sms = 0;
    STA_CUDA_TRY(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, *dev));
    STA_CUDA_TRY(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, *dev));
    STA_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, *dev));
    di.sm100 = (major == 10 && minor == 0);
    di.num_sms = sms;
    di.checked = true;
  }
  return STA_OK;
}

// ------------------------------------------------------------------ TMA maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// [rows, d] bf16 row-major, box of box_rows rows x 64 columns, 128-byte swizzle.
sta_status make_row_map(CUtensorMap* map, const void* base, int64_t rows, int d,
                        int box_rows = 128) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return STA_ERR_CUDA;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(d) * 2};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? STA_OK : STA_ERR_CUDA;
}

// Raster-ordered [slices, T, H, W, d] bf16 viewed as (d, W, H, T, slice) with
// slice stride S*d (the text rows sit between slices); box = one 128-row block
// of a tile: {64, cw, bh, bt, 1} with cw*bh*bt = 128, 128-byte swizzle.
sta_status make_raster_map(CUtensorMap* map, const void* base, int slices, int S, int T,
                           int H, int W, int d, int cw, int bh, int bt) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return STA_ERR_CUDA;
  const cuuint64_t e = 2;
  cuuint64_t dims[5] = {cuuint64_t(d), cuuint64_t(W), cuuint64_t(H), cuuint64_t(T),
                        cuuint64_t(slices)};
  cuuint64_t strides[4] = {e * d, e * d * W, e * d * W * H, e * d * S};
  cuuint32_t box[5] = {64, cuuint32_t(cw), cuuint32_t(bh), cuuint32_t(bt), 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? STA_OK : STA_ERR_CUDA;
}

// ------------------------------------------------------------------ geometry
struct Geom {
  int T, H, W, ct, ch, cw;
  int NT, NH, NW, NV, V, Lv, S;
  bool has_text;
  int text_len;
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

sta_status make_geom(Geom* g, int T, int H, int W, const int tile[3], int has_text,
                     int text_len) {
  if (tile == nullptr) return STA_ERR_INVALID_ARG;
  if (T < 1 || H < 1 || W < 1) return STA_ERR_INVALID_ARG;
  if (tile[0] < 1 || tile[1] < 1 || tile[2] < 1) return STA_ERR_INVALID_ARG;
  if (T % tile[0] || H % tile[1] || W % tile[2]) return STA_ERR_INVALID_ARG;
  if (has_text != 0 && has_text != 1) return STA_ERR_INVALID_ARG;
  const int64_t lv = static_cast<int64_t>(T) * H * W;
  if (lv + STA_TEXT_PAD > (int64_t(1) << 30)) return STA_ERR_INVALID_ARG;
  g->T = T; g->H = H; g->W = W;
  g->ct = tile[0]; g->ch = tile[1]; g->cw = tile[2];
  g->NT = T / tile[0]; g->NH = H / tile[1]; g->NW = W / tile[2];
  g->NV = g->NT * g->NH * g->NW;
  g->V = tile[0] * tile[1] * tile[2];
  g->Lv = static_cast<int>(lv);
  g->has_text = has_text != 0;
  g->S = g->Lv + (g->has_text ? STA_TEXT_PAD : 0);
  g->text_len = g->has_text ? text_len : 0;
  if (g->has_text && (text_len < 0 || text_len > STA_TEXT_PAD)) return STA_ERR_INVALID_ARG;
  return STA_OK;
}

void window_range_host(int c, int w, int n, int* s, int* e) {
  *e = std::min(w, n);
  *s = c - *e / 2;
  if (*s < 0) *s = 0;
  if (*s > n - *e) *s = n - *e;
}

// Raster-order kernels load every 128-row block of a tile as one box
// {cw, bh, bt} of whole tile rows: cw | 128 and (ch*cw | 128 or 128 | ch*cw).
bool raster_boxes_ok(const Geom& g) {
  const int plane = g.ch * g.cw;
  return 128 % g.cw == 0 && (128 % plane == 0 || plane % 128 == 0);
}

sta_status check_windows(const int* window, int heads) {
  if (window == nullptr) return STA_ERR_INVALID_ARG;
  for (int h = 0; h < heads; ++h)
    for (int a = 0; a < 3; ++a)
      if (window[3 * h + a] < 1) return STA_ERR_INVALID_ARG;
  return STA_OK;
}

// Window classes: distinct windows, heads mapped onto them in first-seen order.
struct Classes {
  std::vector<int> head_class;
  std::vector<int> win;   // [nclass][3]
  int nclass = 0;
};

Classes make_classes(const int* window, int heads) {
  Classes c;
  c.head_class.resize(heads);
  for (int h = 0; h < heads; ++h) {
    int found = -1;
    for (int k = 0; k < c.nclass; ++k)
      if (c.win[3 * k] == window[3 * h] && c.win[3 * k + 1] == window[3 * h + 1] &&
          c.win[3 * k + 2] == window[3 * h + 2]) {
        found = k;
        break;
      }
    if (found < 0) {
      found = c.nclass++;
      c.win.insert(c.win.end(), {window[3 * h], window[3 * h + 1], window[3 * h + 2]});
    }
    c.head_class[h] = found;
  }
  return c;
}

int class_video_tiles(const Geom& g, const int* w) {
  return std::min(w[0], g.NT) * std::min(w[1], g.NH) * std::min(w[2], g.NW);
}

void launch_lists(int* counts, int* ids, const Classes& cls, const Geom& g, int max_k,
                  cudaStream_t st, bool token_mode = false) {
  sta::ListWindows wp;
  std::memset(&wp, 0, sizeof(wp));
  std::memcpy(wp.w, cls.win.data(), sizeof(int) * cls.win.size());
  sta::ListGeom lg;
  lg.NT = g.NT; lg.NH = g.NH; lg.NW = g.NW; lg.NV = g.NV;
  lg.NQ = g.NV + (g.has_text ? 1 : 0);
  lg.max_k = max_k;
  lg.text_block = (g.has_text && g.text_len > 0) ? 1 : 0;
  lg.token_mode = token_mode ? 1 : 0;
  lg.ct = g.ct; lg.ch = g.ch; lg.cw = g.cw;
  const int total = cls.nclass * lg.NQ;
  const int threads = 128;
  sta::kv_tile_list_kernel<<<(total + threads - 1) / threads, threads, 0, st>>>(
      counts, ids, wp, cls.nclass, lg);
}

// Token-window mode (3-D sliding window): key tiles covering the windows of
// the tokens of query tile c along one axis (same rule as the list kernel).
void token_tile_range_host(int c, int w, int cs, int n, int* s, int* e) {
  const int X = n * cs;
  const int we = std::min(w, X);
  const int lo = std::max(0, std::min(c * cs - we / 2, X - we));
  const int hi = std::max(0, std::min(c * cs + cs - 1 - we / 2, X - we));
  *s = lo / cs;
  *e = (hi + we - 1) / cs - *s + 1;
}

// (start, extent) of query tile t's key-tile box along the three axes.
void tile_box(const Geom& g, const int* w, int t, bool token_mode, int st[3], int ex[3]) {
  const int c[3] = {t / (g.NW * g.NH), (t / g.NW) % g.NH, t % g.NW};
  const int n[3] = {g.NT, g.NH, g.NW};
  const int cs[3] = {g.ct, g.ch, g.cw};
  for (int a = 0; a < 3; ++a) {
    if (token_mode)
      token_tile_range_host(c[a], w[a], cs[a], n[a], &st[a], &ex[a]);
    else
      window_range_host(c[a], w[a], n[a], &st[a], &ex[a]);
  }
}

// ------------------------------------------------------------------ stream order
// A library-owned device buffer (workspace) that calls on different streams
// share: every call that writes it first waits, on the GPU, for the last call
// that used it when that call came on another stream, and records an event
// after its own launches.  Calls on one stream are ordered by the stream
// itself and pay nothing.  A call made while its stream is being captured
// into a CUDA graph neither waits nor records (event work across a capture
// boundary is not allowed); such calls are ordered by their own stream only.
struct StreamOrder {
  cudaEvent_t ev = nullptr;
  cudaStream_t last = nullptr;
  bool used = false;
};

bool stream_capturing(cudaStream_t st) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) return false;
  return cs != cudaStreamCaptureStatusNone;
}

sta_status order_begin(StreamOrder& o, cudaStream_t st) {
  if (!o.used || o.last == st || stream_capturing(st)) return STA_OK;
  STA_CUDA_TRY(cudaStreamWaitEvent(st, o.ev, 0));
  return STA_OK;
}

sta_status order_end(StreamOrder& o, cudaStream_t st) {
  if (stream_capturing(st)) return STA_OK;
  if (o.ev == nullptr) STA_CUDA_TRY(cudaEventCreateWithFlags(&o.ev, cudaEventDisableTiming));
  STA_CUDA_TRY(cudaEventRecord(o.ev, st));
  o.last = st;
  o.used = true;
  return STA_OK;
}

// ------------------------------------------------------------------ workspace
struct Workspace {
  void* buf = nullptr;
  size_t cap = 0;
  std::string plan_key;     // key of the plan currently resident in `buf`
  std::vector<WorkItem> items;
  std::vector<int> item_off;  // CTA-pair plans: first item of each cluster, + end
  StreamOrder order;
};
Workspace g_ws[64];

sta_status ensure_workspace(int dev, size_t bytes) {
  Workspace& w = g_ws[dev];
  if (w.cap >= bytes) return STA_OK;
  if (w.buf != nullptr) {
    STA_CUDA_TRY(cudaFree(w.buf));
    w.buf = nullptr;
    w.cap = 0;
  }
  size_t cap = std::max<size_t>(bytes, size_t(1) << 20);
  STA_CUDA_TRY(cudaMalloc(&w.buf, cap));
  w.cap = cap;
  w.plan_key.clear();
  return STA_OK;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ------------------------------------------------------------------ STA plan
// Work items pair two 128-row query blocks with the same key-tile list so
// both slots of a CTA share every K/V load.  Blocks of one tile pair up;
// with an odd number of blocks per tile the leftover blocks of tiles whose
// windows start at the same tile (hence have identical lists) pair up; the
// text query block (256 rows) is one pair.  Items are ordered longest first
// (text items, then by list length) and, within one length, by slice so that
// concurrently running CTAs share K/V in L2.
std::vector<WorkItem> plan_sta(const Geom& g, const Classes& cls, int B, int heads,
                               int max_k, std::vector<int>* lengths, bool token_mode = false) {
  const int NQ = g.NV + (g.has_text ? 1 : 0);
  const int bpt = g.V / sta::kBM;
  const int text_blocks = (g.text_len + sta::kBN - 1) / sta::kBN;
  const int sentinel = (g.has_text && g.text_len > 0) ? 1 : 0;
  struct Entry { int len; int slice; WorkItem it; };
  std::vector<Entry> all;
  for (int b = 0; b < B; ++b) {
    for (int h = 0; h < heads; ++h) {
      const int slice = b * heads + h;
      const int base = slice * g.S;
      const int c = cls.head_class[h];
      const int* w = &cls.win[3 * c];
      std::map<int64_t, int> pending;   // key-tile box -> leftover block row
      for (int t = 0; t < g.NV; ++t) {
        int bs[3], be[3];
        tile_box(g, w, t, token_mode, bs, be);
        const int vlen = be[0] * be[1] * be[2] * bpt + sentinel * text_blocks;
        const int list = c * NQ + t;
        const int row0 = base + t * g.V;
        int qb = 0;
        for (; qb + 1 < bpt; qb += 2)
          all.push_back({vlen, slice, {row0 + qb * sta::kBM, row0 + (qb + 1) * sta::kBM, base, list}});
        if (qb < bpt) {
          // identical boxes give identical lists: pair the leftover blocks
          int64_t key = 0;
          for (int a = 0; a < 3; ++a) key = key * 4096 + bs[a];
          for (int a = 0; a < 3; ++a) key = key * 4096 + be[a];
          auto itp = pending.find(key);
          if (itp == pending.end()) {
            pending[key] = t;
          } else {
            const int t0 = itp->second;
            pending.erase(itp);
            all.push_back({vlen, slice,
                           {base + t0 * g.V + qb * sta::kBM, row0 + qb * sta::kBM, base,
                            c * NQ + t0}});
          }
        }
      }
      for (auto& kv : pending) {
        const int t0 = kv.second;
        int bs[3], be[3];
        tile_box(g, w, t0, token_mode, bs, be);
        const int vlen = be[0] * be[1] * be[2] * bpt + sentinel * text_blocks;
        all.push_back({vlen, slice, {base + t0 * g.V + (bpt - 1) * sta::kBM, -1, base, c * NQ + t0}});
      }
      if (g.has_text) {
        const int tlen = g.NV * bpt + sentinel * text_blocks;
        all.push_back({tlen, slice, {base + g.Lv, base + g.Lv + sta::kBM, base, c * NQ + g.NV}});
      }
    }
  }
  std::stable_sort(all.begin(), all.end(), [](const Entry& a, const Entry& b) {
    if (a.len != b.len) return a.len > b.len;
    return a.slice < b.slice;
  });
  std::vector<WorkItem> items;
  items.reserve(all.size());
  if (lengths) lengths->clear();
  for (auto& e : all) {
    items.push_back(e.it);
    if (lengths) lengths->push_back(e.len);
  }
  (void)max_k;
  return items;
}

// Persistent CTA-pair kernel: items (sorted longest first) go, one at a time,
// to the cluster with the least work so far (longest-processing-time-first);
// equal lengths thus go round robin, so clusters running at the same time
// work on neighbouring items.  Returns the items cluster by cluster and, in
// *off, the first item of each cluster followed by the total.
std::vector<WorkItem> assign_to_clusters(const std::vector<WorkItem>& items,
                                         const std::vector<int>& lengths, int nclusters,
                                         std::vector<int>* off) {
  const int nc = std::max(1, std::min(nclusters, static_cast<int>(items.size())));
  std::vector<std::vector<int>> per(nc);
  using Load = std::pair<int64_t, int>;
  std::priority_queue<Load, std::vector<Load>, std::greater<Load>> heap;
  for (int c = 0; c < nc; ++c) heap.push({0, c});
  for (size_t i = 0; i < items.size(); ++i) {
    Load l = heap.top();
    heap.pop();
    per[l.second].push_back(static_cast<int>(i));
    l.first += lengths[i];
    heap.push(l);
  }
  std::vector<WorkItem> out;
  out.reserve(items.size());
  off->assign(1, 0);
  for (int c = 0; c < nc; ++c) {
    for (int i : per[c]) out.push_back(items[i]);
    off->push_back(static_cast<int>(out.size()));
  }
  return out;
}

std::string sta_key(int dev, int B, int heads, int d, const Geom& g, const int* window) {
  std::string k = "sta:" + std::to_string(dev) + ":" + std::to_string(B) + ":" +
                  std::to_string(heads) + ":" + std::to_string(d) + ":" + std::to_string(g.T) +
                  "," + std::to_string(g.H) + "," + std::to_string(g.W) + ":" +
                  std::to_string(g.ct) + "," + std::to_string(g.ch) + "," +
                  std::to_string(g.cw) + ":" + std::to_string(g.has_text) + ":" +
                  std::to_string(g.text_len) + ":";
  for (int i = 0; i < 3 * heads; ++i) k += std::to_string(window[i]) + ",";
  return k;
}

// mq5/mk5/mv5: 5-D maps of raster-ordered tensors (R), else unused copies.
template <int D, Mode M, bool R = false>
sta_status launch_attn(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                       const FwdParams& prm, int num_items, cudaStream_t st,
                       const CUtensorMap* mq5 = nullptr, const CUtensorMap* mk5 = nullptr,
                       const CUtensorMap* mv5 = nullptr) {
  constexpr int smem = sta::FwdCfg<D>::kSmemBytes;
  static bool attr_set[64] = {};
  int dev = 0;
  STA_CUDA_TRY(cudaGetDevice(&dev));
  if (!attr_set[dev]) {
    STA_CUDA_TRY(cudaFuncSetAttribute(sta::attn_fwd_kernel<D, M, R>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
    attr_set[dev] = true;
  }
  sta::attn_fwd_kernel<D, M, R><<<num_items, sta::kFwdThreads, smem, st>>>(
      mq, mk, mv, mq5 ? *mq5 : mq, mk5 ? *mk5 : mk, mv5 ? *mv5 : mv, prm);
  STA_CUDA_TRY(cudaGetLastError());
  return STA_OK;
}

// The d = 128 STA kernel on CTA pairs (attn_fwd_pair.cuh): one cluster of two
// CTAs per work item.
template <bool R>
sta_status launch_attn_pair(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                            const FwdParams& prm, int num_items, cudaStream_t st,
                            const CUtensorMap* mq5, const CUtensorMap* mk5,
                            const CUtensorMap* mv5) {
  constexpr int smem = sta::PairCfg::kSmemBytes;
  static bool attr_set[64] = {};
  int dev = 0;
  STA_CUDA_TRY(cudaGetDevice(&dev));
  if (!attr_set[dev]) {
    STA_CUDA_TRY(cudaFuncSetAttribute(sta::attn_fwd_pair_kernel<R>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
    attr_set[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * static_cast<unsigned>(num_items), 1, 1);
  cfg.blockDim = dim3(sta::kPairThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  STA_CUDA_TRY(cudaLaunchKernelEx(&cfg, sta::attn_fwd_pair_kernel<R>, mq, mk, mv,
                                  mq5 ? *mq5 : mq, mk5 ? *mk5 : mk, mv5 ? *mv5 : mv, prm));
  return STA_OK;
}

// Kernel choice for d = 128 STA: 0 = the one-SM kernel (the default; also
// the kernel of d = 64 and of the masked modes), 1 = the CTA-pair kernel
// when the geometry allows (opt-in: on the video+text workload it is as fast
// on tile-ordered inputs and slower on raster-ordered ones, its K / V loads
// taking longer to land than its three score buffers cover).
int g_pair_mode = 0;

sta_status forward_impl(const void* q, const void* k, const void* v, void* out, float* lse,
                        int B, int heads, int d, int T, int H, int W, const int tile[3],
                        const int* window, int text_len, int has_text, void* stream,
                        bool raster = false, const int* token_window = nullptr) {
  // token_window != nullptr: token-level 3-D sliding window (one window of
  // tokens for every head) instead of STA's window of tiles.
  const bool token_mode = token_window != nullptr;
  int tok_wins[3 * kMaxClasses];
  if (token_mode) {
    if (heads > kMaxClasses) return STA_ERR_UNSUPPORTED;
    for (int a = 0; a < 3; ++a)
      if (token_window[a] < 1) return STA_ERR_INVALID_ARG;
    for (int h = 0; h < heads; ++h)
      for (int a = 0; a < 3; ++a) tok_wins[3 * h + a] = token_window[a];
    window = tok_wins;
  }
  if (!q || !k || !v || !out) return STA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return STA_ERR_INVALID_ARG;
  if (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)) return STA_ERR_INVALID_ARG;
  if (B < 1 || heads < 1) return STA_ERR_INVALID_ARG;
  if (out == q || out == k || out == v) return STA_ERR_INVALID_ARG;
  Geom g;
  sta_status s = make_geom(&g, T, H, W, tile, has_text, text_len);
  if (s != STA_OK) return s;
  s = check_windows(window, heads);
  if (s != STA_OK) return s;
  if (d != 64 && d != 128) return STA_ERR_UNSUPPORTED;
  if (g.V % sta::kBM != 0) return STA_ERR_UNSUPPORTED;
  if (token_mode && (g.ch != 8 || g.cw != 8)) return STA_ERR_UNSUPPORTED;
  const int64_t total_rows = int64_t(B) * heads * g.S;
  if (total_rows >= (int64_t(1) << 31)) return STA_ERR_INVALID_ARG;
  // Raster order: a 128-row block of a tile must be a box {cw, bh, bt} of
  // whole rows of the tile (cw | 128, and ch*cw | 128 or 128 | ch*cw).
  int box_h = 0, box_t = 0;
  if (raster) {
    if (!raster_boxes_ok(g)) return STA_ERR_UNSUPPORTED;
    box_h = std::min(g.ch, 128 / g.cw);
    box_t = 128 / (g.cw * box_h);
    if (B * int64_t(heads) > (int64_t(1) << 31)) return STA_ERR_INVALID_ARG;
  }
  int dev = 0;
  s = current_device(&dev);
  if (s != STA_OK) return s;
  if (!g_dev[dev].sm100) return STA_ERR_UNSUPPORTED;

  std::lock_guard<std::mutex> lock(g_mu);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  Classes cls = make_classes(window, heads);
  if (cls.nclass > kMaxClasses) return STA_ERR_UNSUPPORTED;
  const int sentinel = (g.has_text && g.text_len > 0) ? 1 : 0;
  int max_k = 1;
  for (int c = 0; c < cls.nclass; ++c) {
    if (token_mode) {
      for (int t = 0; t < g.NV; ++t) {
        int bs[3], be[3];
        tile_box(g, &cls.win[3 * c], t, true, bs, be);
        max_k = std::max(max_k, be[0] * be[1] * be[2] + sentinel);
      }
    } else {
      max_k = std::max(max_k, class_video_tiles(g, &cls.win[3 * c]) + sentinel);
    }
  }
  if (g.has_text) max_k = std::max(max_k, g.NV + sentinel);
  const int NQ = g.NV + (g.has_text ? 1 : 0);
  const size_t counts_bytes = align_up(sizeof(int) * size_t(cls.nclass) * NQ, 256);
  const size_t ids_bytes = align_up(sizeof(int) * size_t(cls.nclass) * NQ * max_k, 256);

  // CTA pairs (attn_fwd_pair.cuh) for d = 128 STA; in raster order each CTA
  // loads 64-row halves of the key blocks, so a block's box must split into
  // two boxes (along t, else along h).
  const bool khalf_t = box_t >= 2;
  const bool pair = g_pair_mode == 1 && d == 128 && !token_mode &&
                    (!raster || khalf_t || box_h % 2 == 0);
  const int nclusters_max = std::max(1, g_dev[dev].num_sms / 2);

  const std::string key = std::string(token_mode ? "tok:" : "") + (pair ? "pair:" : "") +
                          sta_key(dev, B, heads, d, g, window);
  Workspace& ws = g_ws[dev];
  std::vector<WorkItem> fresh;
  std::vector<int> fresh_off;
  const bool cached = (ws.plan_key == key && ws.buf != nullptr);
  if (!cached) {
    std::vector<int> lengths;
    fresh = plan_sta(g, cls, B, heads, max_k, &lengths, token_mode);
    if (pair) {
      // slice-major (longest first within a slice), so that the clusters
      // running at the same time read the keys / values of one or two heads
      std::vector<int> idx(fresh.size());
      for (size_t i = 0; i < idx.size(); ++i) idx[i] = static_cast<int>(i);
      std::stable_sort(idx.begin(), idx.end(), [&](int a, int b) {
        const int sa = fresh[a].kv_base / g.S, sb = fresh[b].kv_base / g.S;
        if (sa != sb) return sa < sb;
        return lengths[a] > lengths[b];
      });
      std::vector<WorkItem> by_slice;
      std::vector<int> len_by_slice;
      for (int i : idx) {
        by_slice.push_back(fresh[i]);
        len_by_slice.push_back(lengths[i]);
      }
      fresh = assign_to_clusters(by_slice, len_by_slice, nclusters_max, &fresh_off);
    }
  }
  const std::vector<WorkItem>& items = cached ? ws.items : fresh;
  const std::vector<int>& offs = cached ? ws.item_off : fresh_off;
  const size_t items_bytes = align_up(sizeof(WorkItem) * items.size(), 256);
  const size_t off_bytes = sizeof(int) * offs.size();
  s = ensure_workspace(dev, counts_bytes + ids_bytes + items_bytes + off_bytes);
  if (s != STA_OK) return s;
  s = order_begin(ws.order, st);
  if (s != STA_OK) return s;
  uint8_t* wbuf = static_cast<uint8_t*>(ws.buf);
  int* d_counts = reinterpret_cast<int*>(wbuf);
  int* d_ids = reinterpret_cast<int*>(wbuf + counts_bytes);
  WorkItem* d_items = reinterpret_cast<WorkItem*>(wbuf + counts_bytes + ids_bytes);
  int* d_off = reinterpret_cast<int*>(wbuf + counts_bytes + ids_bytes + items_bytes);
  if (ws.plan_key != key) {
    ws.items = std::move(fresh);
    ws.item_off = std::move(fresh_off);
    STA_CUDA_TRY(cudaMemcpyAsync(d_items, ws.items.data(), sizeof(WorkItem) * ws.items.size(),
                                 cudaMemcpyHostToDevice, st));
    if (!ws.item_off.empty())
      STA_CUDA_TRY(cudaMemcpyAsync(d_off, ws.item_off.data(), sizeof(int) * ws.item_off.size(),
                                   cudaMemcpyHostToDevice, st));
    ws.plan_key = key;
  }
  // one CTA per item, or (pairs) one persistent cluster per item list
  const int num_items = pair ? static_cast<int>(ws.item_off.size()) - 1
                             : static_cast<int>(ws.items.size());

  CUtensorMap mq, mk, mv;
  s = make_row_map(&mq, q, total_rows, d);
  if (s == STA_OK) s = make_row_map(&mk, k, total_rows, d);
  if (s == STA_OK) s = make_row_map(&mv, v, total_rows, d);
  if (s != STA_OK) return s;

  // a2: tile lists, rebuilt on every call.
  launch_lists(d_counts, d_ids, cls, g, max_k, st, token_mode);
  STA_CUDA_TRY(cudaGetLastError());

  FwdParams prm{};
  prm.items = d_items;
  prm.item_off = pair ? d_off : nullptr;
  prm.dbg_rows_q = static_cast<int>(total_rows);
  prm.dbg_rows_kv = static_cast<int>(total_rows);
  prm.dbg_lists = cls.nclass * NQ;
  prm.counts = d_counts;
  prm.ids = d_ids;
  prm.max_k = max_k;
  prm.tile_blocks = g.V / sta::kBM;
  prm.V = g.V;
  prm.L_v = g.Lv;
  prm.text_len = g.text_len;
  prm.text_blocks = (g.text_len + sta::kBN - 1) / sta::kBN;
  prm.text_sentinel = sentinel;
  prm.window = 0;
  prm.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(double(d)));
  prm.out = static_cast<__nv_bfloat16*>(out);
  prm.lse = lse;
  prm.rg.S = g.S;
  prm.rg.ct = g.ct; prm.rg.ch = g.ch; prm.rg.cw = g.cw;
  prm.rg.H = g.H; prm.rg.W = g.W;
  prm.rg.NH = g.NH; prm.rg.NW = g.NW;
  prm.rg.T = g.T;
  if (token_mode)
    for (int a = 0; a < 3; ++a) prm.win3[a] = token_window[a];
  prm.khalf_t = khalf_t ? 1 : 0;
  prm.kbox_t = box_t;
  prm.kbox_h = box_h;
  CUtensorMap mk_half;
  if (pair) {
    s = make_row_map(&mk_half, k, total_rows, d, 64);
    if (s != STA_OK) return s;
  }
  auto dispatch = [&]() -> sta_status {
    if (raster) {
      CUtensorMap q5, k5, v5;
      const int slices = B * heads;
      sta_status r = make_raster_map(&q5, q, slices, g.S, g.T, g.H, g.W, d, g.cw, box_h, box_t);
      if (r == STA_OK && pair)
        r = make_raster_map(&k5, k, slices, g.S, g.T, g.H, g.W, d, g.cw,
                            khalf_t ? box_h : box_h / 2, khalf_t ? box_t / 2 : box_t);
      else if (r == STA_OK)
        r = make_raster_map(&k5, k, slices, g.S, g.T, g.H, g.W, d, g.cw, box_h, box_t);
      if (r == STA_OK)
        r = make_raster_map(&v5, v, slices, g.S, g.T, g.H, g.W, d, g.cw, box_h, box_t);
      if (r != STA_OK) return r;
      if (pair) return launch_attn_pair<true>(mq, mk_half, mv, prm, num_items, st, &q5, &k5, &v5);
      if (token_mode) {
        if (d == 128)
          return launch_attn<128, Mode::kSwa3d, true>(mq, mk, mv, prm, num_items, st, &q5, &k5,
                                                       &v5);
        return launch_attn<64, Mode::kSwa3d, true>(mq, mk, mv, prm, num_items, st, &q5, &k5,
                                                    &v5);
      }
      if (d == 128)
        return launch_attn<128, Mode::kSta, true>(mq, mk, mv, prm, num_items, st, &q5, &k5, &v5);
      return launch_attn<64, Mode::kSta, true>(mq, mk, mv, prm, num_items, st, &q5, &k5, &v5);
    }
    if (token_mode) return STA_ERR_UNSUPPORTED;
    if (pair)
      return launch_attn_pair<false>(mq, mk_half, mv, prm, num_items, st, nullptr, nullptr,
                                     nullptr);
    if (d == 128) return launch_attn<128, Mode::kSta>(mq, mk, mv, prm, num_items, st);
    return launch_attn<64, Mode::kSta>(mq, mk, mv, prm, num_items, st);
  };
  s = dispatch();
  if (s != STA_OK) return s;
  return order_end(ws.order, st);
}

// ------------------------------------------------------------------ host-buffer pipeline
// sta_forward_raster_host: q, k, v and out live in host memory.  The (batch,
// head) slices are independent problems, so the call walks them in chunks of
// whole heads through two device staging buffers: the copy-in of chunk c+1
// (stream s_in), the attention of chunk c (the caller's stream) and the
// copy-out of chunk c-1 (stream s_out) run at the same time.
struct HostPipe {
  bool ready = false;
  bool used = false;
  cudaStream_t s_in = nullptr, s_out = nullptr;
  cudaEvent_t start = nullptr, end = nullptr;
  cudaEvent_t in_ready[2] = {}, comp_done[2] = {}, out_done[2] = {};
  void* buf = nullptr;   // [2 buffers][q, k, v, out][chunk bytes]
  size_t cap = 0;
};
HostPipe g_pipe[64];
std::mutex g_pipe_mu;

sta_status host_pipe_setup(HostPipe& hp, size_t bytes) {
  if (!hp.ready) {
    STA_CUDA_TRY(cudaStreamCreateWithFlags(&hp.s_in, cudaStreamNonBlocking));
    STA_CUDA_TRY(cudaStreamCreateWithFlags(&hp.s_out, cudaStreamNonBlocking));
    cudaEvent_t* evs[] = {&hp.start, &hp.end, &hp.in_ready[0], &hp.in_ready[1],
                          &hp.comp_done[0], &hp.comp_done[1], &hp.out_done[0],
                          &hp.out_done[1]};
    for (cudaEvent_t* e : evs) STA_CUDA_TRY(cudaEventCreateWithFlags(e, cudaEventDisableTiming));
    hp.ready = true;
  }
  if (hp.cap < bytes) {
    if (hp.buf != nullptr) {
      // the previous call's copies may still read or write the old buffer
      STA_CUDA_TRY(cudaEventSynchronize(hp.end));
      STA_CUDA_TRY(cudaFree(hp.buf));
      hp.buf = nullptr;
      hp.cap = 0;
    }
    STA_CUDA_TRY(cudaMalloc(&hp.buf, bytes));
    hp.cap = bytes;
  }
  return STA_OK;
}

sta_status forward_host_impl(const void* q, const void* k, const void* v, void* out, int B,
                             int heads, int d, int T, int H, int W, const int tile[3],
                             const int* window, int text_len, int has_text,
                             size_t chunk_bytes_max, void* stream) {
  if (!q || !k || !v || !out) return STA_ERR_INVALID_ARG;
  if (B < 1 || heads < 1) return STA_ERR_INVALID_ARG;
  if (out == q || out == k || out == v) return STA_ERR_INVALID_ARG;
  if (chunk_bytes_max == 0) chunk_bytes_max = STA_HOST_CHUNK_BYTES;
  Geom g;
  sta_status s = make_geom(&g, T, H, W, tile, has_text, text_len);
  if (s != STA_OK) return s;
  s = check_windows(window, heads);
  if (s != STA_OK) return s;
  if (d != 64 && d != 128) return STA_ERR_UNSUPPORTED;
  if (g.V % sta::kBM != 0 || !raster_boxes_ok(g)) return STA_ERR_UNSUPPORTED;
  if (make_classes(window, heads).nclass > kMaxClasses) return STA_ERR_UNSUPPORTED;
  int dev = 0;
  s = current_device(&dev);
  if (s != STA_OK) return s;
  if (!g_dev[dev].sm100) return STA_ERR_UNSUPPORTED;

  const size_t slice_bytes = size_t(g.S) * d * sizeof(__nv_bfloat16);
  const int hc = static_cast<int>(std::max<size_t>(
      1, std::min<size_t>(size_t(heads), chunk_bytes_max / slice_bytes)));
  const size_t chunk_bytes = size_t(hc) * slice_bytes;

  std::lock_guard<std::mutex> lock(g_pipe_mu);
  HostPipe& hp = g_pipe[dev];
  s = host_pipe_setup(hp, 8 * chunk_bytes);
  if (s != STA_OK) return s;
  uint8_t* base = static_cast<uint8_t*>(hp.buf);
  auto staged = [&](int buf, int tensor) { return base + (buf * 4 + tensor) * chunk_bytes; };
  const uint8_t* src[3] = {static_cast<const uint8_t*>(q), static_cast<const uint8_t*>(k),
                           static_cast<const uint8_t*>(v)};
  uint8_t* dst = static_cast<uint8_t*>(out);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

  // Everything earlier on the caller's stream, and every copy of the previous
  // call (which may have come on another stream), precedes this call.
  STA_CUDA_TRY(cudaEventRecord(hp.start, st));
  STA_CUDA_TRY(cudaStreamWaitEvent(hp.s_in, hp.start, 0));
  STA_CUDA_TRY(cudaStreamWaitEvent(hp.s_out, hp.start, 0));
  if (hp.used) {
    STA_CUDA_TRY(cudaStreamWaitEvent(hp.s_in, hp.end, 0));
    STA_CUDA_TRY(cudaStreamWaitEvent(st, hp.end, 0));
  }
  hp.used = true;
  int c = 0;
  for (int b = 0; b < B; ++b) {
    for (int h0 = 0; h0 < heads; h0 += hc, ++c) {
      const int n = std::min(hc, heads - h0);
      const int buf = c & 1;
      const size_t off = (size_t(b) * heads + h0) * slice_bytes;
      const size_t bytes = size_t(n) * slice_bytes;
      // inputs of buffer `buf` are free once chunk c-2's attention has run
      if (c >= 2) STA_CUDA_TRY(cudaStreamWaitEvent(hp.s_in, hp.comp_done[buf], 0));
      for (int t = 0; t < 3; ++t)
        STA_CUDA_TRY(cudaMemcpyAsync(staged(buf, t), src[t] + off, bytes,
                                     cudaMemcpyHostToDevice, hp.s_in));
      STA_CUDA_TRY(cudaEventRecord(hp.in_ready[buf], hp.s_in));
      STA_CUDA_TRY(cudaStreamWaitEvent(st, hp.in_ready[buf], 0));
      // its output is free once chunk c-2 has been copied out
      if (c >= 2) STA_CUDA_TRY(cudaStreamWaitEvent(st, hp.out_done[buf], 0));
      s = forward_impl(staged(buf, 0), staged(buf, 1), staged(buf, 2), staged(buf, 3),
                       nullptr, 1, n, d, T, H, W, tile, window + 3 * h0, text_len, has_text,
                       st, true);
      if (s != STA_OK) return s;
      STA_CUDA_TRY(cudaEventRecord(hp.comp_done[buf], st));
      STA_CUDA_TRY(cudaStreamWaitEvent(hp.s_out, hp.comp_done[buf], 0));
      STA_CUDA_TRY(cudaMemcpyAsync(dst + off, staged(buf, 3), bytes, cudaMemcpyDeviceToHost,
                                   hp.s_out));
      STA_CUDA_TRY(cudaEventRecord(hp.out_done[buf], hp.s_out));
    }
  }
  // the caller's stream completes only after the last byte of out is home
  STA_CUDA_TRY(cudaEventRecord(hp.end, hp.s_out));
  STA_CUDA_TRY(cudaStreamWaitEvent(st, hp.end, 0));
  return STA_OK;
}

template <int kVec>
void launch_permute(const void* in, void* out, const sta::ReorderGeom& rg, int slices,
                    int to_tile, cudaStream_t st) {
  dim3 grid(rg.num_tiles + (rg.S > rg.Lv ? 1 : 0), slices);
  sta::tile_permute_kernel<kVec><<<grid, 256, 0, st>>>(
      static_cast<const uint4*>(in), static_cast<uint4*>(out), rg, to_tile);
}

sta_status permute_impl(const void* in, void* out, int B, int heads, int d, int T, int H,
                        int W, const int tile[3], int has_text, void* stream, int to_tile) {
  if (!in || !out || in == out) return STA_ERR_INVALID_ARG;
  if (!aligned16(in) || !aligned16(out)) return STA_ERR_INVALID_ARG;
  if (B < 1 || heads < 1 || d < 1) return STA_ERR_INVALID_ARG;
  if (B * static_cast<int64_t>(heads) > 65535) return STA_ERR_INVALID_ARG;
  Geom g;
  sta_status s = make_geom(&g, T, H, W, tile, has_text, 0);
  if (s != STA_OK) return s;
  const int vec = d * 2 / 16;
  if ((d * 2) % 16 != 0) return STA_ERR_UNSUPPORTED;
  if (vec != 4 && vec != 8 && vec != 16 && vec != 32) return STA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(g.V) * vec >= (int64_t(1) << 31)) return STA_ERR_INVALID_ARG;
  int dev = 0;
  s = current_device(&dev);
  if (s != STA_OK) return s;
  sta::ReorderGeom rg;
  rg.T = g.T; rg.H = g.H; rg.W = g.W;
  rg.ct = g.ct; rg.ch = g.ch; rg.cw = g.cw;
  rg.NH = g.NH; rg.NW = g.NW;
  rg.V = g.V; rg.S = g.S; rg.Lv = g.Lv; rg.num_tiles = g.NV;
  rg.div_cw = sta::make_fastdiv(g.cw);
  rg.div_chcw = sta::make_fastdiv(g.ch * g.cw);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int slices = B * heads;
  switch (vec) {
    case 4: launch_permute<4>(in, out, rg, slices, to_tile, st); break;
    case 8: launch_permute<8>(in, out, rg, slices, to_tile, st); break;
    case 16: launch_permute<16>(in, out, rg, slices, to_tile, st); break;
    default: launch_permute<32>(in, out, rg, slices, to_tile, st); break;
  }
  STA_CUDA_TRY(cudaGetLastError());
  return STA_OK;
}

// ------------------------------------------------------------------ SWA plan
std::vector<WorkItem> plan_swa(int B, int hq, int hkv, int S, int window) {
  const int group = hq / hkv;
  const int nqb = S / sta::kBM;
  struct Entry { int len; int kvs; WorkItem it; };
  std::vector<Entry> all;
  for (int b = 0; b < B; ++b)
    for (int hk = 0; hk < hkv; ++hk) {
      const int kv_base = (b * hkv + hk) * S;
      for (int qb = 0; qb < nqb; ++qb) {
        const int lo = qb * sta::kBN - window + 1;
        const int kb_lo = lo <= 0 ? 0 : lo / sta::kBN;
        const int len = qb - kb_lo + 1;
        for (int g0 = 0; g0 < group; g0 += 2) {
          const int h0 = hk * group + g0;
          const int q0 = (b * hq + h0) * S + qb * sta::kBM;
          const int q1 = (g0 + 1 < group) ? (b * hq + h0 + 1) * S + qb * sta::kBM : -1;
          all.push_back({len, b * hkv + hk, {q0, q1, kv_base, qb}});
        }
      }
    }
  std::stable_sort(all.begin(), all.end(), [](const Entry& a, const Entry& b) {
    if (a.len != b.len) return a.len > b.len;
    return a.kvs < b.kvs;
  });
  std::vector<WorkItem> items;
  for (auto& e : all) items.push_back(e.it);
  return items;
}

// ------------------------------------------------------------------ no-alloc
// Fixed scratch for sta_forward_noalloc: tile lists and the work plan live in
// this file-scope array instead of the lazily grown workspace.  Host code must
// not pass `g_noalloc_scratch` itself to a kernel (on the host it names a
// stand-in, not device memory): each device's address is looked up once with
// cudaGetSymbolAddress while that device is current.
static __device__ __align__(256) unsigned char g_noalloc_scratch[STA_NOALLOC_SCRATCH_BYTES];

struct NoAllocState {
  bool ready = false;
  unsigned char* scratch = nullptr;   // device address of g_noalloc_scratch
  std::string plan_key;               // host-side plan cache (host memory only)
  std::vector<WorkItem> items;
  // Key of the plan whose items are in the device array.  Only this entry
  // point writes the array, so an unchanged key means the items are there.
  std::string resident_key;
};
NoAllocState g_noalloc[64];

sta_status forward_noalloc_impl(const void* q, const void* k, const void* v, void* out,
                                int B, int heads, int d, int T, int H, int W,
                                const int tile[3], const int* window, int text_len,
                                int has_text, void* stream) {
  if (!q || !k || !v || !out) return STA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return STA_ERR_INVALID_ARG;
  if (B < 1 || heads < 1) return STA_ERR_INVALID_ARG;
  if (out == q || out == k || out == v) return STA_ERR_INVALID_ARG;
  Geom g;
  sta_status s = make_geom(&g, T, H, W, tile, has_text, text_len);
  if (s != STA_OK) return s;
  s = check_windows(window, heads);
  if (s != STA_OK) return s;
  if (d != 64 && d != 128) return STA_ERR_UNSUPPORTED;
  if (g.V % sta::kBM != 0) return STA_ERR_UNSUPPORTED;
  const int64_t total_rows = int64_t(B) * heads * g.S;
  if (total_rows >= (int64_t(1) << 31)) return STA_ERR_INVALID_ARG;
  Classes cls = make_classes(window, heads);
  if (cls.nclass > kMaxClasses) return STA_ERR_UNSUPPORTED;
  const int sentinel = (g.has_text && g.text_len > 0) ? 1 : 0;
  int max_k = 1;
  for (int c = 0; c < cls.nclass; ++c)
    max_k = std::max(max_k, class_video_tiles(g, &cls.win[3 * c]) + sentinel);
  if (g.has_text) max_k = std::max(max_k, g.NV + sentinel);
  const int NQ = g.NV + (g.has_text ? 1 : 0);
  const size_t counts_bytes = align_up(sizeof(int) * size_t(cls.nclass) * NQ, 256);
  const size_t ids_bytes = align_up(sizeof(int) * size_t(cls.nclass) * NQ * max_k, 256);
  // Size check from the geometry alone, before any plan is built.
  const int bpt = g.V / sta::kBM;
  const size_t max_items = size_t(B) * heads * (size_t(g.NV) * ((bpt + 1) / 2) + 1);
  if (counts_bytes + ids_bytes + sizeof(WorkItem) * max_items > STA_NOALLOC_SCRATCH_BYTES)
    return STA_ERR_SCRATCH_LIMIT;
  int dev = 0;
  s = current_device(&dev);
  if (s != STA_OK) return s;
  if (!g_dev[dev].sm100) return STA_ERR_UNSUPPORTED;

  std::lock_guard<std::mutex> lock(g_mu);
  NoAllocState& na = g_noalloc[dev];
  if (!na.ready) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr)
      return STA_ERR_CUDA;
    na.scratch = static_cast<unsigned char*>(ptr);
    na.ready = true;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const std::string key = sta_key(dev, B, heads, d, g, window);
  if (na.plan_key != key) {
    na.items = plan_sta(g, cls, B, heads, max_k, nullptr);
    na.plan_key = key;
  }
  const size_t items_bytes = sizeof(WorkItem) * na.items.size();
  if (counts_bytes + ids_bytes + items_bytes > STA_NOALLOC_SCRATCH_BYTES)
    return STA_ERR_SCRATCH_LIMIT;
  int* d_counts = reinterpret_cast<int*>(na.scratch);
  int* d_ids = reinterpret_cast<int*>(na.scratch + counts_bytes);
  WorkItem* d_items = reinterpret_cast<WorkItem*>(na.scratch + counts_bytes + ids_bytes);

  CUtensorMap mq, mk, mv;
  s = make_row_map(&mq, q, total_rows, d);
  if (s == STA_OK) s = make_row_map(&mk, k, total_rows, d);
  if (s == STA_OK) s = make_row_map(&mv, v, total_rows, d);
  if (s != STA_OK) return s;
  // The array keeps the previous call's contents: the plan is copied in only
  // when it differs from the one already there, and the list kernel rewrites
  // every count and id that the attention kernel reads.
  if (na.resident_key != key) {
    na.resident_key.clear();
    STA_CUDA_TRY(cudaMemcpyAsync(d_items, na.items.data(), items_bytes, cudaMemcpyHostToDevice,
                                 st));
    na.resident_key = key;
  }
  launch_lists(d_counts, d_ids, cls, g, max_k, st);
  STA_CUDA_TRY(cudaGetLastError());

  FwdParams prm{};
  prm.items = d_items;
  prm.item_off = nullptr;
  prm.dbg_rows_q = static_cast<int>(total_rows);
  prm.dbg_rows_kv = static_cast<int>(total_rows);
  prm.dbg_lists = cls.nclass * NQ;
  prm.counts = d_counts;
  prm.ids = d_ids;
  prm.max_k = max_k;
  prm.tile_blocks = bpt;
  prm.V = g.V;
  prm.L_v = g.Lv;
  prm.text_len = g.text_len;
  prm.text_blocks = (g.text_len + sta::kBN - 1) / sta::kBN;
  prm.text_sentinel = sentinel;
  prm.window = 0;
  prm.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(double(d)));
  prm.out = static_cast<__nv_bfloat16*>(out);
  prm.lse = nullptr;
  const int num_items = static_cast<int>(na.items.size());
  if (d == 128) return launch_attn<128, Mode::kSta>(mq, mk, mv, prm, num_items, st);
  return launch_attn<64, Mode::kSta>(mq, mk, mv, prm, num_items, st);
}

// ------------------------------------------------------------------ 2-D slide
// Workspace of the 2-D slide-attention path (coordinate table, block
// rectangles, pair lists and plan), separate from the STA workspace.
struct Slide2dWs {
  void* buf = nullptr;
  size_t cap = 0;
  std::string key;
  StreamOrder order;
};
Slide2dWs g_ws2d[64];

int ilog2_exact(int n) {
  int l = 0;
  while ((1 << l) < n) ++l;
  return (1 << l) == n ? l : -1;
}

sta_status slide2d_check(int n, int window, int order) {
  const int l = ilog2_exact(n);
  if (l < 4 || l > 15) return STA_ERR_UNSUPPORTED;  // 16 <= n <= 32768, power of two
  if (window < 1) return STA_ERR_INVALID_ARG;
  if (order != 0 && order != 1) return STA_ERR_INVALID_ARG;
  if (order == 0 && n < 128) return STA_ERR_UNSUPPORTED;  // raster blocks must be row pieces
  return STA_OK;
}

sta_status slide2d_ensure(int dev, size_t bytes) {
  Slide2dWs& w = g_ws2d[dev];
  if (w.cap >= bytes) return STA_OK;
  if (w.buf) {
    STA_CUDA_TRY(cudaFree(w.buf));
    w.buf = nullptr;
    w.cap = 0;
  }
  STA_CUDA_TRY(cudaMalloc(&w.buf, bytes));
  w.cap = bytes;
  w.key.clear();
  return STA_OK;
}

// coords + rects for `order` into the given device buffers.
void launch_coords_rects(uint32_t* coords, int4* rects, int n, int order, cudaStream_t st) {
  const int l = ilog2_exact(n);
  const int N = n * n, nb = N / 128;
  sta::order_coords_kernel<<<(N + 255) / 256, 256, 0, st>>>(coords, l, order);
  sta::block_rect_kernel<<<(nb * 32 + 255) / 256, 256, 0, st>>>(coords, rects, nb);
}

// ------------------------------------------------------------------ backward
struct BwdWs {
  void* buf = nullptr;
  size_t cap = 0;
  StreamOrder order;
};
BwdWs g_wsb[64];

template <int D, bool kDKV>
sta_status launch_bwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                      const CUtensorMap& mdo, const sta::BwdParams& prm, int num_items,
                      cudaStream_t st) {
  // dK/dV: attn_bwd_dkv_kernel (whole streamed blocks); dQ: attn_bwd_dq_kernel (K and V
  // in separate rings, next block's scores during this block's elementwise work)
  constexpr int smem = kDKV ? sta::BwdCfg<D>::kSmemBytes : sta::BwdDqCfg<D>::kSmemBytes;
  static bool attr_set[64] = {};
  int dev = 0;
  STA_CUDA_TRY(cudaGetDevice(&dev));
  if (!attr_set[dev]) {
    if constexpr (kDKV) {
      STA_CUDA_TRY(cudaFuncSetAttribute(sta::attn_bwd_dkv_kernel<D>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
    } else {
      STA_CUDA_TRY(cudaFuncSetAttribute(sta::attn_bwd_dq_kernel<D>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
    }
    attr_set[dev] = true;
  }
  if constexpr (kDKV)
    sta::attn_bwd_dkv_kernel<D><<<num_items, sta::kDkvThreads, smem, st>>>(mq, mk, mv, mdo, prm);
  else
    sta::attn_bwd_dq_kernel<D><<<num_items, sta::kDqThreads, smem, st>>>(mq, mk, mv, mdo, prm);
  STA_CUDA_TRY(cudaGetLastError());
  return STA_OK;
}

sta_status backward_impl(const void* q, const void* k, const void* v, const void* o,
                         const void* dout, const float* lse, void* dq, void* dk, void* dv,
                         int B, int heads, int d, int T, int H, int W, const int tile[3],
                         const int* window, int text_len, int has_text, void* stream) {
  const void* ins[6] = {q, k, v, o, dout, lse};
  for (const void* x : ins)
    if (!x || !aligned16(x)) return STA_ERR_INVALID_ARG;
  const void* outs[3] = {dq, dk, dv};
  for (const void* x : outs) {
    if (!x || !aligned16(x)) return STA_ERR_INVALID_ARG;
    for (const void* y : ins)
      if (x == y) return STA_ERR_INVALID_ARG;
  }
  if (dq == dk || dq == dv || dk == dv || B < 1 || heads < 1) return STA_ERR_INVALID_ARG;
  Geom g;
  sta_status s = make_geom(&g, T, H, W, tile, has_text, text_len);
  if (s != STA_OK) return s;
  s = check_windows(window, heads);
  if (s != STA_OK) return s;
  if (d != 64 && d != 128) return STA_ERR_UNSUPPORTED;
  if (g.V % 128 != 0) return STA_ERR_UNSUPPORTED;
  const int64_t rows = int64_t(B) * heads * g.S;
  if (rows >= (int64_t(1) << 31)) return STA_ERR_INVALID_ARG;
  int dev = 0;
  s = current_device(&dev);
  if (s != STA_OK) return s;
  if (!g_dev[dev].sm100) return STA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  Classes cls = make_classes(window, heads);
  if (cls.nclass > kMaxClasses) return STA_ERR_UNSUPPORTED;
  const int sentinel = (g.has_text && g.text_len > 0) ? 1 : 0;
  const int NQ = g.NV + (g.has_text ? 1 : 0);
  const int max_k = g.NV + 1;   // both list kinds fit in NV + 1 entries
  const int bpt = g.V / 128;
  // workspace: -lse2, -D, forward lists, transposed lists, two plans
  const size_t vb = align_up(sizeof(float) * size_t(rows), 256);
  const size_t cb = align_up(sizeof(int) * size_t(cls.nclass) * NQ, 256);
  const size_t ib = align_up(sizeof(int) * size_t(cls.nclass) * NQ * max_k, 256);
  const size_t blocks = size_t(B) * heads * (g.S / 128);
  const size_t pb = align_up(sizeof(WorkItem) * blocks, 256);
  const size_t total = 2 * vb + 2 * cb + 2 * ib + 2 * pb;
  BwdWs& ws = g_wsb[dev];
  if (ws.cap < total) {
    if (ws.buf) STA_CUDA_TRY(cudaFree(ws.buf));
    ws.buf = nullptr;
    ws.cap = 0;
    STA_CUDA_TRY(cudaMalloc(&ws.buf, total));
    ws.cap = total;
  }
  s = order_begin(ws.order, st);
  if (s != STA_OK) return s;
  uint8_t* w = static_cast<uint8_t*>(ws.buf);
  float* neg_lse2 = reinterpret_cast<float*>(w);
  float* neg_delta = reinterpret_cast<float*>(w + vb);
  int* fc = reinterpret_cast<int*>(w + 2 * vb);
  int* tc = reinterpret_cast<int*>(w + 2 * vb + cb);
  int* fi = reinterpret_cast<int*>(w + 2 * vb + 2 * cb);
  int* ti = reinterpret_cast<int*>(w + 2 * vb + 2 * cb + ib);
  WorkItem* qitems = reinterpret_cast<WorkItem*>(w + 2 * vb + 2 * cb + 2 * ib);
  WorkItem* kitems = reinterpret_cast<WorkItem*>(w + 2 * vb + 2 * cb + 2 * ib + pb);
  // plans: one item per 128-row block, longest streams first
  std::vector<std::pair<int, WorkItem>> qp, kp;
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < heads; ++h) {
      const int base = (b * heads + h) * g.S;
      const int c = cls.head_class[h];
      const int* wv = &cls.win[3 * c];
      const int qlen = class_video_tiles(g, wv) * bpt + sentinel * ((g.text_len + 127) / 128);
      for (int t = 0; t < g.NV; ++t)
        for (int sb = 0; sb < bpt; ++sb) {
          const int row = base + t * g.V + sb * 128;
          qp.push_back({qlen, {row, -1, base, c * NQ + t}});
          // key tile t is seen by the query tiles whose box holds it
          int seen = 1;
          for (int a = 0; a < 3; ++a) {
            const int cc = a == 0 ? t / (g.NW * g.NH) : (a == 1 ? (t / g.NW) % g.NH : t % g.NW);
            const int na = a == 0 ? g.NT : (a == 1 ? g.NH : g.NW);
            int cntq = 0;
            for (int x = 0; x < na; ++x) {
              int s0, e0;
              window_range_host(x, wv[a], na, &s0, &e0);
              cntq += (cc >= s0 && cc < s0 + e0);
            }
            seen *= cntq;
          }
          kp.push_back({seen * bpt + (g.has_text ? 2 : 0), {row, -1, base, c * NQ + t}});
        }
      if (g.has_text) {
        const int qtext = g.NV * bpt + sentinel * ((g.text_len + 127) / 128);
        for (int tb = 0; tb < 2; ++tb) {
          const int row = base + g.Lv + tb * 128;
          qp.push_back({qtext, {row, -1, base, c * NQ + g.NV}});
          kp.push_back({g.NV * bpt + 2, {row, -1, base, c * NQ + g.NV}});
        }
      }
    }
  auto by_len = [](const std::pair<int, WorkItem>& a, const std::pair<int, WorkItem>& b) {
    return a.first > b.first;
  };
  std::stable_sort(qp.begin(), qp.end(), by_len);
  // dK/dV: stream lengths differ from key tile to key tile (border tiles lie
  // in more windows), so a global longest-first order would interleave the
  // (batch, head) slices and the CTAs running at once would stream every
  // slice's Q and dO through L2.  The text key blocks (every query block of
  // their slice, the longest items by far) go first, so that none of them
  // starts near the end; then the video key blocks slice by slice, longest
  // first inside a slice.
  auto by_slice_len = [&](const std::pair<int, WorkItem>& a, const std::pair<int, WorkItem>& b) {
    const bool ta = a.second.list % NQ == g.NV, tb = b.second.list % NQ == g.NV;
    if (ta != tb) return ta;
    if (a.second.kv_base != b.second.kv_base) return a.second.kv_base < b.second.kv_base;
    return a.first > b.first;
  };
  std::stable_sort(kp.begin(), kp.end(), by_slice_len);
  std::vector<WorkItem> qv, kv;
  for (auto& e : qp) qv.push_back(e.second);
  for (auto& e : kp) kv.push_back(e.second);
  STA_CUDA_TRY(cudaMemcpyAsync(qitems, qv.data(), sizeof(WorkItem) * qv.size(),
                               cudaMemcpyHostToDevice, st));
  STA_CUDA_TRY(cudaMemcpyAsync(kitems, kv.data(), sizeof(WorkItem) * kv.size(),
                               cudaMemcpyHostToDevice, st));
  // -D and -lse2
  const long long warps = (rows * (d / 8) + 31) / 32;
  const int pre_blocks = static_cast<int>((warps * 32 + 255) / 256);
  if (d == 128)
    sta::bwd_preprocess_kernel<128><<<pre_blocks, 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dout), lse,
        neg_delta, neg_lse2, rows);
  else
    sta::bwd_preprocess_kernel<64><<<pre_blocks, 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dout), lse,
        neg_delta, neg_lse2, rows);
  // forward and transposed tile lists
  launch_lists(fc, fi, cls, g, max_k, st);
  {
    sta::ListWindows wp;
    std::memset(&wp, 0, sizeof(wp));
    std::memcpy(wp.w, cls.win.data(), sizeof(int) * cls.win.size());
    sta::ListGeom lg;
    std::memset(&lg, 0, sizeof(lg));
    lg.NT = g.NT; lg.NH = g.NH; lg.NW = g.NW; lg.NV = g.NV; lg.NQ = NQ; lg.max_k = max_k;
    const int tot = cls.nclass * NQ;
    sta::kv_tile_list_transposed_kernel<<<(tot + 127) / 128, 128, 0, st>>>(
        tc, ti, wp, cls.nclass, lg, g.has_text ? 1 : 0);
  }
  STA_CUDA_TRY(cudaGetLastError());
  CUtensorMap mq, mk, mv, mdo;
  s = make_row_map(&mq, q, rows, d);
  if (s == STA_OK) s = make_row_map(&mk, k, rows, d);
  if (s == STA_OK) s = make_row_map(&mv, v, rows, d);
  if (s == STA_OK) s = make_row_map(&mdo, dout, rows, d);
  if (s != STA_OK) return s;
  sta::BwdParams prm;
  std::memset(&prm, 0, sizeof(prm));
  prm.max_k = max_k;
  prm.tile_blocks = bpt;
  prm.V = g.V;
  prm.L_v = g.Lv;
  prm.text_len = g.text_len;
  prm.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(double(d)));
  prm.scale = static_cast<float>(1.0 / std::sqrt(double(d)));
  prm.neg_lse2 = neg_lse2;
  prm.neg_delta = neg_delta;
  prm.dbg_rows = static_cast<int>(rows);
  prm.dbg_lists = cls.nclass * NQ;
  // dQ: forward lists, text key blocks with valid keys
  prm.items = qitems;
  prm.counts = fc;
  prm.ids = fi;
  prm.text_sentinel = sentinel;
  prm.text_blocks = (g.text_len + 127) / 128;
  prm.out_a = static_cast<__nv_bfloat16*>(dq);
  prm.out_b = nullptr;
  s = d == 128 ? launch_bwd<128, false>(mq, mk, mv, mdo, prm, int(qv.size()), st)
               : launch_bwd<64, false>(mq, mk, mv, mdo, prm, int(qv.size()), st);
  if (s != STA_OK) return s;
  // dK, dV: transposed lists, the 256 text query rows as two blocks
  prm.items = kitems;
  prm.counts = tc;
  prm.ids = ti;
  prm.text_sentinel = g.has_text ? 1 : 0;
  prm.text_blocks = 2;
  prm.out_a = static_cast<__nv_bfloat16*>(dk);
  prm.out_b = static_cast<__nv_bfloat16*>(dv);
  s = d == 128 ? launch_bwd<128, true>(mq, mk, mv, mdo, prm, int(kv.size()), st)
               : launch_bwd<64, true>(mq, mk, mv, mdo, prm, int(kv.size()), st);
  if (s != STA_OK) return s;
  return order_end(ws.order, st);
}

}  // namespace

// ====================================================================== C ABI
extern "C" {

const char* sta_status_string(sta_status s) {
  switch (s) {
    case STA_OK: return "STA_OK";
    case STA_ERR_INVALID_ARG: return "STA_ERR_INVALID_ARG: argument rejected";
    case STA_ERR_UNSUPPORTED: return "STA_ERR_UNSUPPORTED: shape or device not supported";
    case STA_ERR_CUDA: return "STA_ERR_CUDA: a CUDA call failed";
    case STA_ERR_DEVICE_TIMEOUT: return "STA_ERR_DEVICE_TIMEOUT: a device wait gave up";
    case STA_ERR_SCRATCH_LIMIT:
      return "STA_ERR_SCRATCH_LIMIT: problem needs more than the fixed no-alloc scratch";
    case STA_ERR_DEVICE_BOUNDS:
      return "STA_ERR_DEVICE_BOUNDS: a device bounds check failed (debug build)";
  }
  return "STA_ERR_UNKNOWN";
}

sta_status sta_tile_reorder(const void* in, void* out, int B, int heads, int d, int T, int H,
                            int W, const int tile[3], int has_text, void* stream) {
  return permute_impl(in, out, B, heads, d, T, H, W, tile, has_text, stream, 1);
}

sta_status sta_tile_unreorder(const void* in, void* out, int B, int heads, int d, int T,
                              int H, int W, const int tile[3], int has_text, void* stream) {
  return permute_impl(in, out, B, heads, d, T, H, W, tile, has_text, stream, 0);
}

sta_status sta_build_kv_tile_lists(int* counts, int* ids, int max_k, int heads, int T, int H,
                                   int W, const int tile[3], const int* window, int text_len,
                                   int has_text, void* stream) {
  if (!counts || !ids || heads < 1 || heads > kMaxClasses) return STA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(counts) & 3u) || (reinterpret_cast<uintptr_t>(ids) & 3u))
    return STA_ERR_INVALID_ARG;
  Geom g;
  sta_status s = make_geom(&g, T, H, W, tile, has_text, text_len);
  if (s != STA_OK) return s;
  s = check_windows(window, heads);
  if (s != STA_OK) return s;
  const int sentinel = (g.has_text && g.text_len > 0) ? 1 : 0;
  int need = 1;
  for (int h = 0; h < heads; ++h)
    need = std::max(need, class_video_tiles(g, &window[3 * h]) + sentinel);
  if (g.has_text) need = std::max(need, g.NV + sentinel);
  if (max_k < need) return STA_ERR_INVALID_ARG;
  int dev = 0;
  s = current_device(&dev);
  if (s != STA_OK) return s;
  // one class per head: the public lists are per head
  Classes cls;
  cls.nclass = heads;
  cls.win.assign(window, window + 3 * heads);
  cls.head_class.resize(heads);
  for (int h = 0; h < heads; ++h) cls.head_class[h] = h;
  launch_lists(counts, ids, cls, g, max_k, reinterpret_cast<cudaStream_t>(stream));
  STA_CUDA_TRY(cudaGetLastError());
  return STA_OK;
}

sta_status sta_forward(const void* q, const void* k, const void* v, void* out, int B,
                       int heads, int d, int T, int H, int W, const int tile[3],
                       const int* window, int text_len, int has_text, void* stream) {
  return forward_impl(q, k, v, out, nullptr, B, heads, d, T, H, W, tile, window, text_len,
                      has_text, stream);
}

sta_status sta_forward_raster(const void* q, const void* k, const void* v, void* out,
                              float* lse, int B, int heads, int d, int T, int H, int W,
                              const int tile[3], const int* window, int text_len, int has_text,
                              void* stream) {
  return forward_impl(q, k, v, out, lse, B, heads, d, T, H, W, tile, window, text_len,
                      has_text, stream, true);
}

sta_status sta_swa3d_forward(const void* q, const void* k, const void* v, void* out, int B,
                             int heads, int d, int T, int H, int W, const int tile[3],
                             const int window_tokens[3], int text_len, int has_text,
                             void* stream) {
  if (window_tokens == nullptr) return STA_ERR_INVALID_ARG;
  return forward_impl(q, k, v, out, nullptr, B, heads, d, T, H, W, tile, window_tokens,
                      text_len, has_text, stream, true, window_tokens);
}

sta_status sta_forward_noalloc(const void* q, const void* k, const void* v, void* out, int B,
                               int heads, int d, int T, int H, int W, const int tile[3],
                               const int* window, int text_len, int has_text, void* stream) {
  return forward_noalloc_impl(q, k, v, out, B, heads, d, T, H, W, tile, window, text_len,
                              has_text, stream);
}

sta_status sta_forward_lse(const void* q, const void* k, const void* v, void* out, float* lse,
                           int B, int heads, int d, int T, int H, int W, const int tile[3],
                           const int* window, int text_len, int has_text, void* stream) {
  if (lse == nullptr) return STA_ERR_INVALID_ARG;
  return forward_impl(q, k, v, out, lse, B, heads, d, T, H, W, tile, window, text_len,
                      has_text, stream);
}

sta_status sta_swa_forward(const void* q, const void* k, const void* v, void* out, int B,
                           int hq, int hkv, int d, int S, int window, int causal,
                           void* stream) {
  if (!q || !k || !v || !out) return STA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return STA_ERR_INVALID_ARG;
  if (out == q || out == k || out == v) return STA_ERR_INVALID_ARG;
  if (B < 1 || hq < 1 || hkv < 1 || hq % hkv != 0 || S < 1 || window < 1) return STA_ERR_INVALID_ARG;
  if (causal != 1) return STA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return STA_ERR_UNSUPPORTED;
  if (S % sta::kBM != 0) return STA_ERR_UNSUPPORTED;
  const int64_t qrows = int64_t(B) * hq * S;
  if (qrows >= (int64_t(1) << 31)) return STA_ERR_INVALID_ARG;
  int dev = 0;
  sta_status s = current_device(&dev);
  if (s != STA_OK) return s;
  if (!g_dev[dev].sm100) return STA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const std::string key = "swa:" + std::to_string(dev) + ":" + std::to_string(B) + ":" +
                          std::to_string(hq) + ":" + std::to_string(hkv) + ":" +
                          std::to_string(S) + ":" + std::to_string(window);
  Workspace& ws = g_ws[dev];
  std::vector<WorkItem> fresh;
  const bool cached = (ws.plan_key == key && ws.buf != nullptr);
  if (!cached) fresh = plan_swa(B, hq, hkv, S, window);
  const size_t bytes = sizeof(WorkItem) * (cached ? ws.items.size() : fresh.size());
  s = ensure_workspace(dev, bytes);
  if (s != STA_OK) return s;
  s = order_begin(ws.order, st);
  if (s != STA_OK) return s;
  WorkItem* d_items = static_cast<WorkItem*>(ws.buf);
  if (ws.plan_key != key) {
    ws.items = std::move(fresh);
    STA_CUDA_TRY(cudaMemcpyAsync(d_items, ws.items.data(), sizeof(WorkItem) * ws.items.size(),
                                 cudaMemcpyHostToDevice, st));
    ws.plan_key = key;
  }
  CUtensorMap mq, mk, mv;
  s = make_row_map(&mq, q, qrows, d);
  if (s == STA_OK) s = make_row_map(&mk, k, int64_t(B) * hkv * S, d);
  if (s == STA_OK) s = make_row_map(&mv, v, int64_t(B) * hkv * S, d);
  if (s != STA_OK) return s;
  FwdParams prm{};
  std::memset(&prm, 0, sizeof(prm));
  prm.items = d_items;
  prm.dbg_rows_q = static_cast<int>(qrows);
  prm.dbg_rows_kv = static_cast<int>(int64_t(B) * hkv * S);
  prm.window = window;
  prm.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(double(d)));
  prm.out = static_cast<__nv_bfloat16*>(out);
  prm.lse = nullptr;
  const int num_items = static_cast<int>(ws.items.size());
  s = d == 128 ? launch_attn<128, Mode::kSwa>(mq, mk, mv, prm, num_items, st)
               : launch_attn<64, Mode::kSwa>(mq, mk, mv, prm, num_items, st);
  if (s != STA_OK) return s;
  return order_end(ws.order, st);
}

int sta_debug_checks(void) { return STA_DEBUG ? 1 : 0; }

sta_status sta_debug_pair_kernel(int pair) {
  if (pair != 0 && pair != 1) return STA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_mu);
  g_pair_mode = pair;
  return STA_OK;
}

sta_status sta_debug_inject(int mode, int wait_limit_ms) {
  if (mode < 0 || mode > 1 || wait_limit_ms < 1) return STA_ERR_INVALID_ARG;
  const unsigned long long limit = static_cast<unsigned long long>(wait_limit_ms) * 1000000ull;
  STA_CUDA_TRY(cudaDeviceSynchronize());
  STA_CUDA_TRY(cudaMemcpyToSymbol(sta::g_inject, &mode, sizeof(mode)));
  STA_CUDA_TRY(cudaMemcpyToSymbol(sta::g_wait_limit_ns, &limit, sizeof(limit)));
  return STA_OK;
}

sta_status sta_hilbert_reorder(const void* in, void* out, int B, int heads, int d, int n,
                               int to_hilbert, void* stream) {
  if (!in || !out || in == out || !aligned16(in) || !aligned16(out)) return STA_ERR_INVALID_ARG;
  if (B < 1 || heads < 1 || d < 1 || (to_hilbert != 0 && to_hilbert != 1)) return STA_ERR_INVALID_ARG;
  const int l = ilog2_exact(n);
  if (l < 1 || l > 15) return STA_ERR_UNSUPPORTED;
  if ((d * 2) % 16 != 0) return STA_ERR_UNSUPPORTED;
  const int vec = d * 2 / 16;
  if (vec != 4 && vec != 8 && vec != 16 && vec != 32) return STA_ERR_UNSUPPORTED;
  int dev = 0;
  sta_status s = current_device(&dev);
  if (s != STA_OK) return s;
  const long long total = static_cast<long long>(B) * heads * n * n * vec;
  const int grid = static_cast<int>(std::min<long long>((total + 255) / 256, 148LL * 64));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const uint4* a = static_cast<const uint4*>(in);
  uint4* b = static_cast<uint4*>(out);
  switch (vec) {
    case 4: sta::hilbert_permute_kernel<4><<<grid, 256, 0, st>>>(a, b, l, total, to_hilbert); break;
    case 8: sta::hilbert_permute_kernel<8><<<grid, 256, 0, st>>>(a, b, l, total, to_hilbert); break;
    case 16: sta::hilbert_permute_kernel<16><<<grid, 256, 0, st>>>(a, b, l, total, to_hilbert); break;
    default: sta::hilbert_permute_kernel<32><<<grid, 256, 0, st>>>(a, b, l, total, to_hilbert); break;
  }
  STA_CUDA_TRY(cudaGetLastError());
  return STA_OK;
}

sta_status sta_build_slide_block_lists(int* counts, int* ids, int* classes, int max_k, int n,
                                       int window, int order, void* stream) {
  if (!counts || !ids) return STA_ERR_INVALID_ARG;
  sta_status s = slide2d_check(n, window, order);
  if (s != STA_OK) return s;
  const int nb = n * n / 128;
  if (max_k < nb) return STA_ERR_INVALID_ARG;
  if (nb > 8192) return STA_ERR_UNSUPPORTED;
  int dev = 0;
  s = current_device(&dev);
  if (s != STA_OK) return s;
  std::lock_guard<std::mutex> lock(g_mu);
  const size_t cbytes = align_up(sizeof(uint32_t) * size_t(n) * n, 256);
  s = slide2d_ensure(dev, cbytes + sizeof(int4) * nb);
  if (s != STA_OK) return s;
  g_ws2d[dev].key.clear();
  uint8_t* w = static_cast<uint8_t*>(g_ws2d[dev].buf);
  uint32_t* coords = reinterpret_cast<uint32_t*>(w);
  int4* rects = reinterpret_cast<int4*>(w + cbytes);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  s = order_begin(g_ws2d[dev].order, st);
  if (s != STA_OK) return s;
  launch_coords_rects(coords, rects, n, order, st);
  const size_t smem = sizeof(int) * (512 + nb);
  sta::slide_block_list_kernel<<<nb, 256, smem, st>>>(counts, ids, classes, max_k, coords, rects,
                                                      nb, n, window, 1);
  STA_CUDA_TRY(cudaGetLastError());
  return order_end(g_ws2d[dev].order, st);
}

sta_status sta_slide2d_forward(const void* q, const void* k, const void* v, void* out, int B,
                               int heads, int d, int n, int window, int order, void* stream) {
  if (!q || !k || !v || !out) return STA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return STA_ERR_INVALID_ARG;
  if (out == q || out == k || out == v || B < 1 || heads < 1) return STA_ERR_INVALID_ARG;
  sta_status s = slide2d_check(n, window, order);
  if (s != STA_OK) return s;
  if (d != 64 && d != 128) return STA_ERR_UNSUPPORTED;
  const int N = n * n, nb = N / 128, np = nb / 2;
  if (nb > 8192) return STA_ERR_UNSUPPORTED;
  const int64_t rows = int64_t(B) * heads * N;
  if (rows >= (int64_t(1) << 31)) return STA_ERR_INVALID_ARG;
  int dev = 0;
  s = current_device(&dev);
  if (s != STA_OK) return s;
  if (!g_dev[dev].sm100) return STA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t cbytes = align_up(sizeof(uint32_t) * size_t(N), 256);
  const size_t rbytes = align_up(sizeof(int4) * size_t(nb), 256);
  const size_t nbytes = align_up(sizeof(int) * size_t(np), 256);
  const size_t ibytes = align_up(sizeof(int) * size_t(np) * nb, 256);
  const size_t pbytes = sizeof(WorkItem) * size_t(B) * heads * np;
  s = slide2d_ensure(dev, cbytes + rbytes + nbytes + ibytes + pbytes);
  if (s != STA_OK) return s;
  Slide2dWs& ws = g_ws2d[dev];
  uint8_t* w = static_cast<uint8_t*>(ws.buf);
  uint32_t* coords = reinterpret_cast<uint32_t*>(w);
  int4* rects = reinterpret_cast<int4*>(w + cbytes);
  int* counts = reinterpret_cast<int*>(w + cbytes + rbytes);
  int* ids = reinterpret_cast<int*>(w + cbytes + rbytes + nbytes);
  WorkItem* items = reinterpret_cast<WorkItem*>(w + cbytes + rbytes + nbytes + ibytes);
  const std::string key = "s2d:" + std::to_string(B) + ":" + std::to_string(heads) + ":" +
                          std::to_string(n) + ":" + std::to_string(order);
  s = order_begin(ws.order, st);
  if (s != STA_OK) return s;
  if (ws.key != key) {
    std::vector<WorkItem> plan;
    plan.reserve(size_t(B) * heads * np);
    for (int sl = 0; sl < B * heads; ++sl)
      for (int pi = 0; pi < np; ++pi)
        plan.push_back({sl * N + 2 * pi * 128, sl * N + (2 * pi + 1) * 128, sl * N, pi});
    STA_CUDA_TRY(cudaMemcpyAsync(items, plan.data(), sizeof(WorkItem) * plan.size(),
                                 cudaMemcpyHostToDevice, st));
    ws.key = key;
  }
  // key-block lists of query-block pairs (union), rebuilt on every call
  launch_coords_rects(coords, rects, n, order, st);
  sta::slide_block_list_kernel<<<np, 256, sizeof(int) * (512 + nb), st>>>(
      counts, ids, nullptr, nb, coords, rects, nb, n, window, 2);
  STA_CUDA_TRY(cudaGetLastError());
  CUtensorMap mq, mk, mv;
  s = make_row_map(&mq, q, rows, d);
  if (s == STA_OK) s = make_row_map(&mk, k, rows, d);
  if (s == STA_OK) s = make_row_map(&mv, v, rows, d);
  if (s != STA_OK) return s;
  FwdParams prm{};
  std::memset(&prm, 0, sizeof(prm));
  prm.items = items;
  prm.dbg_rows_q = static_cast<int>(rows);
  prm.dbg_rows_kv = static_cast<int>(rows);
  prm.dbg_lists = np;
  prm.counts = counts;
  prm.ids = ids;
  prm.max_k = nb;
  prm.tile_blocks = 1;
  prm.V = 128;
  prm.L_v = N;
  prm.coords = coords;
  prm.grid_n = n;
  prm.win2 = window;
  prm.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(double(d)));
  prm.out = static_cast<__nv_bfloat16*>(out);
  const int num_items = B * heads * np;
  s = d == 128 ? launch_attn<128, Mode::kSlide2d>(mq, mk, mv, prm, num_items, st)
               : launch_attn<64, Mode::kSlide2d>(mq, mk, mv, prm, num_items, st);
  if (s != STA_OK) return s;
  return order_end(ws.order, st);
}

sta_status sta_backward(const void* q, const void* k, const void* v, const void* out,
                        const void* dout, const float* lse, void* dq, void* dk, void* dv,
                        int B, int heads, int d, int T, int H, int W, const int tile[3],
                        const int* window, int text_len, int has_text, void* stream) {
  return backward_impl(q, k, v, out, dout, lse, dq, dk, dv, B, heads, d, T, H, W, tile, window,
                       text_len, has_text, stream);
}

sta_status sta_forward_raster_host(const void* q, const void* k, const void* v, void* out,
                                   int B, int heads, int d, int T, int H, int W,
                                   const int tile[3], const int* window, int text_len,
                                   int has_text, size_t chunk_bytes, void* stream) {
  return forward_host_impl(q, k, v, out, B, heads, d, T, H, W, tile, window, text_len,
                           has_text, chunk_bytes, stream);
}

sta_status sta_device_status(void* stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return STA_ERR_CUDA;
  unsigned int word = 0;
  STA_CUDA_TRY(cudaMemcpyFromSymbol(&word, sta::g_error_word, sizeof(word)));
  if (word != 0) {
    const unsigned int zero = 0;
    STA_CUDA_TRY(cudaMemcpyToSymbol(sta::g_error_word, &zero, sizeof(zero)));
    // a failed bounds check (debug build) is the cause of any later time-outs
    return (word & sta::kErrBounds) ? STA_ERR_DEVICE_BOUNDS : STA_ERR_DEVICE_TIMEOUT;
  }
  if (cudaGetLastError() != cudaSuccess) return STA_ERR_CUDA;
  return STA_OK;
}

void sta_shutdown(void) {
  std::lock_guard<std::mutex> lock(g_mu);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return;
  // cudaFree waits for the device, so no kernel still reads a buffer
  auto drop_event = [](StreamOrder& o) {
    if (o.ev != nullptr) cudaEventDestroy(o.ev);
    o = StreamOrder();
  };
  for (int i = 0; i < 64; ++i) {
    if (g_ws[i].buf != nullptr || g_ws[i].order.ev != nullptr) {
      cudaSetDevice(i);
      if (g_ws[i].buf != nullptr) cudaFree(g_ws[i].buf);
      drop_event(g_ws[i].order);
      g_ws[i] = Workspace();
    }
    if (g_wsb[i].buf != nullptr || g_wsb[i].order.ev != nullptr) {
      cudaSetDevice(i);
      if (g_wsb[i].buf != nullptr) cudaFree(g_wsb[i].buf);
      drop_event(g_wsb[i].order);
      g_wsb[i] = BwdWs();
    }
    if (g_ws2d[i].buf != nullptr || g_ws2d[i].order.ev != nullptr) {
      cudaSetDevice(i);
      if (g_ws2d[i].buf != nullptr) cudaFree(g_ws2d[i].buf);
      drop_event(g_ws2d[i].order);
      g_ws2d[i] = Slide2dWs();
    }
  }
  {
    std::lock_guard<std::mutex> plock(g_pipe_mu);
    for (int i = 0; i < 64; ++i) {
      HostPipe& hp = g_pipe[i];
      if (!hp.ready) continue;
      cudaSetDevice(i);
      cudaEventSynchronize(hp.end);
      if (hp.buf != nullptr) cudaFree(hp.buf);
      cudaStreamDestroy(hp.s_in);
      cudaStreamDestroy(hp.s_out);
      cudaEvent_t evs[] = {hp.start, hp.end, hp.in_ready[0], hp.in_ready[1], hp.comp_done[0],
                           hp.comp_done[1], hp.out_done[0], hp.out_done[1]};
      for (cudaEvent_t e : evs) cudaEventDestroy(e);
      hp = HostPipe();
    }
  }
  cudaSetDevice(dev);
}

int64_t sta_retained_pairs(int B, int heads, int T, int H, int W, const int tile[3],
                           const int* window, int text_len, int has_text) {
  Geom g;
  if (make_geom(&g, T, H, W, tile, has_text, text_len) != STA_OK) return -1;
  if (B < 1 || heads < 1 || check_windows(window, heads) != STA_OK) return -1;
  int64_t total = 0;
  for (int h = 0; h < heads; ++h) {
    const int64_t vid = class_video_tiles(g, &window[3 * h]);
    int64_t per = int64_t(g.NV) * g.V * (vid * g.V + (g.has_text ? g.text_len : 0));
    if (g.has_text) per += int64_t(STA_TEXT_PAD) * (g.Lv + g.text_len);
    total += per;
  }
  return total * B;
}

}  // extern "C"
