/*
 * sta.h - C ABI of libsta.so: Sliding Tile Attention (STA) forward on B200.
 *
 * Method: the STA README ("Sliding Tile Atteniton Kernel", FastVideo
 * sta_kernel/thunderkitten), sections "Usage", "How Does STA Work?" and
 * "Why is STA Fast?".  A (T,H,W) video token grid is cut into tiles of
 * (ct,ch,cw) tokens (the page's tiles are (6, 8, 8)); every query tile
 * attends to the whole key tiles inside a window of (wt,wh,ww) tiles (the
 * window is counted in tiles), centred on the query tile and shifted inward at
 * the grid border so it always spans the full window; a text block padded to
 * 256 tokens may follow the video (text_length 0..256).
 * Video queries also attend to the first text_len text keys; text queries
 * attend to every video key and the first text_len text keys.  The attention
 * map is therefore made of fully dense or fully empty tile blocks.
 *
 * Conventions for every entry point:
 *  - Tensors are caller-owned device memory, bf16, contiguous
 *    [B, heads, S, d] with S = T*H*W + (has_text ? 256 : 0), base pointers
 *    16-byte aligned.  Nothing is freed or retained by the library.
 *  - `stream` is a cudaStream_t passed as void*; all work is enqueued on it,
 *    asynchronously, with no implicit synchronisation.  NULL = legacy stream.
 *  - Arguments are checked on the host before any launch; on an error status
 *    nothing has been enqueued and no output byte has been written.
 *  - `tile` and `window` are HOST pointers to int32 triples.
 *  - Outputs must not alias inputs.
 *  - Device-side waits are bounded: a kernel that gives up records
 *    STA_ERR_DEVICE_TIMEOUT in a device flag, read by sta_device_status().
 *  - The library keeps lazily grown device workspaces per device (tile
 *    lists and work plans of the forward, backward and 2-D entry points).
 *    A call that writes a workspace first waits, on the GPU, for the last
 *    call that used it if that call came on another stream (an event per
 *    workspace), so calls on several streams are ordered in the order the
 *    host made them; calls on one stream pay nothing for this.  Calls made
 *    while their stream is being captured into a CUDA graph are ordered by
 *    that stream only.  sta_shutdown() releases the workspaces.
 */
#ifndef STA_H_
#define STA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum sta_status {
  STA_OK = 0,
  STA_ERR_INVALID_ARG = 1,    /* shape, window, text or pointer argument rejected  */
  STA_ERR_UNSUPPORTED = 2,    /* legal STA but not built: d not in {64,128},
                                 tile volume not a multiple of 128, not sm_100   */
  STA_ERR_CUDA = 3,           /* a CUDA runtime / driver call failed             */
  STA_ERR_DEVICE_TIMEOUT = 4, /* a bounded device wait gave up (see above)       */
  STA_ERR_SCRATCH_LIMIT = 5,  /* sta_forward_noalloc: the problem needs more than
                                 STA_NOALLOC_SCRATCH_BYTES of scratch            */
  STA_ERR_DEVICE_BOUNDS = 6   /* debug build only: a device bounds check failed  */
} sta_status;

/* Text block size (README Usage: the text block is padded to 256 tokens). */
#define STA_TEXT_PAD 256

/*
 * sta_tile_reorder - raster -> tile token order (README Usage, "a tile is a
 * cube"; tiles must be contiguous rows for the blocks of "Why is STA Fast?"
 * to be dense).  Video row r = (t*H + h)*W + w moves to row
 * tile_id*V + in_tile, tile_id = ((t/ct)*NH + h/ch)*NW + w/cw,
 * in_tile = ((t%ct)*ch + h%ch)*cw + w%cw, V = ct*ch*cw.  Text rows are copied
 * unchanged.  in/out: [B, heads, S, d] bf16 device, d in {64,128}
 * (any d with d*2 % 16 == 0 is accepted).  Bit-exact copy.
 */
sta_status sta_tile_reorder(const void* in, void* out, int B, int heads, int d,
                            int T, int H, int W, const int tile[3],
                            int has_text, void* stream);

/* sta_tile_unreorder - inverse of sta_tile_reorder (tile -> raster order). */
sta_status sta_tile_unreorder(const void* in, void* out, int B, int heads,
                              int d, int T, int H, int W, const int tile[3],
                              int has_text, void* stream);

/*
 * sta_build_kv_tile_lists - per-query-tile KV tile lists (README Usage,
 * "window_size in tiles": one (wt,wh,ww) per head).
 *   counts: device int32 [heads][NQ], NQ = NV + (has_text ? 1 : 0),
 *           NV = (T/ct)*(H/ch)*(W/cw)
 *   ids:    device int32 [heads][NQ][max_k]
 * Row r < NV: ascending ids of the key tiles inside query tile r's window,
 * then the text sentinel NV when has_text && text_len > 0.  Row NV (text
 * queries, only when has_text): 0..NV-1, then NV when text_len > 0.  Unused
 * slots are -1.  window: HOST int32 [heads][3], each entry >= 1 (a window
 * longer than the grid covers the axis).  max_k must be >= the longest row,
 * else STA_ERR_INVALID_ARG.  Integer, bit-exact.
 */
sta_status sta_build_kv_tile_lists(int* counts, int* ids, int max_k, int heads,
                                   int T, int H, int W, const int tile[3],
                                   const int* window, int text_len,
                                   int has_text, void* stream);

/*
 * sta_forward - fused STA attention, tile-ordered q,k,v -> out.
 * Defining passages: README "Usage" (the call
 * sliding_tile_attention(q, k, v, window_size, text_length, has_text): one
 * window of tiles per head, text padded to 256 tokens of which text_length
 * are valid) and "Why is STA Fast?" (a query tile attends to whole key tiles,
 * so every 128 x 128 block of the attention map is fully dense or fully
 * empty; only the padded text columns need a mask).  Output row i is
 * sum_j softmax_j(q_i . k_j / sqrt(d)) v_j over the allowed keys j.
 *   q, k, v: [B, heads, S, d] bf16 device, TILE order (sta_tile_reorder)
 *   out:     [B, heads, S, d] bf16 device, tile order
 *   d in {64, 128}; tile volume ct*ch*cw a multiple of 128;
 *   window: HOST int32 [heads][3]; 0 <= text_len <= 256 (ignored when
 *   has_text == 0).  Scale 1/sqrt(d).  bf16 inputs, fp32 accumulation and
 *   softmax, probabilities rounded to bf16 for the P.V product, output
 *   rounded to nearest even.  Runs on sm_100 only (tcgen05 / TMEM / TMA).
 * Errors: STA_ERR_INVALID_ARG (null or unaligned pointers, aliasing, shape,
 * window or text_len out of range), STA_ERR_UNSUPPORTED (d, tile volume,
 * device), STA_ERR_CUDA; all checked before anything is enqueued.
 */
sta_status sta_forward(const void* q, const void* k, const void* v, void* out,
                       int B, int heads, int d, int T, int H, int W,
                       const int tile[3], const int* window, int text_len,
                       int has_text, void* stream);

/* sta_forward_lse - sta_forward (same passages: README "Usage" and "Why is
 * STA Fast?", same arguments and errors) that also writes the natural-log
 * log-sum-exp of every query row, ln sum_j exp(q_i . k_j / sqrt(d)) over the
 * allowed keys, to `lse` (device fp32 [B, heads, S], 4-byte aligned; the
 * saved statistic of the backward pass). */
sta_status sta_forward_lse(const void* q, const void* k, const void* v,
                           void* out, float* lse, int B, int heads, int d,
                           int T, int H, int W, const int tile[3],
                           const int* window, int text_len, int has_text,
                           void* stream);

/*
 * sta_forward_raster - sta_forward on RASTER-ordered tensors, the README's
 * calling convention (Usage: q, k, v [batch, heads, T*H*W + 256, head_dim]
 * in video order), with the raster <-> tile permutation fused into the
 * attention kernel: each 128-row block of a tile is loaded as a box of the
 * (T, H, W) grid by a 5-D TMA descriptor, and every output row is stored at
 * its raster position.  Same arguments and numerics as sta_forward_lse;
 * `lse` may be NULL (else device fp32 [B, heads, S], raster order).
 * Requires cw | 128 and (ch*cw | 128 or 128 | ch*cw), else
 * STA_ERR_UNSUPPORTED (use sta_tile_reorder + sta_forward + unreorder).
 */
sta_status sta_forward_raster(const void* q, const void* k, const void* v,
                              void* out, float* lse, int B, int heads, int d,
                              int T, int H, int W, const int tile[3],
                              const int* window, int text_len, int has_text,
                              void* stream);

/* Default staging chunk of sta_forward_raster_host: whole heads of up to
 * this many bytes per tensor (at least one head). */
#define STA_HOST_CHUNK_BYTES (64u << 20)

/*
 * sta_forward_raster_host - sta_forward_raster on HOST buffers (same
 * README Usage call, same arguments, layout and numerics; no lse).
 * q, k, v, out: host bf16 [B, heads, S, d], raster order; page-locked
 * (cudaHostAlloc / cudaHostRegister) for the copies to overlap, pageable
 * memory works but serialises.  The (batch, head) slices are independent, so
 * the call moves them in chunks of whole heads (at most `chunk_bytes` per
 * tensor, at least one head; 0 = STA_HOST_CHUNK_BYTES) through two
 * library-owned device staging buffers: copy-in of the
 * next chunk, attention of the current one and copy-out of the previous one
 * overlap on two internal streams and `stream`.  Asynchronous: `out` is
 * complete once `stream` has reached this point (e.g. after
 * cudaStreamSynchronize(stream)); q, k, v must stay unchanged until then.
 * The staging buffers (8 chunks, 2 x {q,k,v,out}) grow on demand and are
 * released by sta_shutdown(); calls on one device are serialised by the
 * library (a later call waits, on the GPU, for the earlier one's copies).
 * Errors: as sta_forward_raster; checked before anything is enqueued, except
 * STA_ERR_CUDA from a failing copy or launch, which may leave `out` partly
 * written.
 */
sta_status sta_forward_raster_host(const void* q, const void* k, const void* v,
                                   void* out, int B, int heads, int d, int T,
                                   int H, int W, const int tile[3],
                                   const int* window, int text_len,
                                   int has_text, size_t chunk_bytes,
                                   void* stream);

/*
 * sta_backward - gradients of sta_forward (STA backward pass; the pages give
 * the forward only, the backward is its gradient).  All tensors TILE order,
 * [B, heads, S, d] bf16 device: q, k, v, out (the forward output), dout
 * (gradient of the loss w.r.t. out); lse: device fp32 [B, heads, S] from
 * sta_forward_lse.  Writes dq, dk, dv (bf16, same layout; caller-owned,
 * distinct from the inputs).  With P = softmax(q k^T / sqrt(d)) on allowed
 * pairs and D = rowsum(dout * out): dv = P^T dout, dS = P (dout v^T - D),
 * dq = dS k / sqrt(d), dk = dS^T q / sqrt(d); padded text keys get zero.
 * fp32 accumulation in tensor memory, P and dS rounded to bf16 for the MMAs.
 * Same geometry limits as sta_forward.
 */
sta_status sta_backward(const void* q, const void* k, const void* v,
                        const void* out, const void* dout, const float* lse,
                        void* dq, void* dk, void* dv, int B, int heads, int d,
                        int T, int H, int W, const int tile[3],
                        const int* window, int text_len, int has_text,
                        void* stream);

/*
 * sta_swa_forward - token-level sliding-window attention with grouped-query
 * heads, the mixed-block baseline of README "Why is STA Fast?"; the 1-D
 * causal window over the previous `window` positions (self included) with
 * GQA follows the sliding-window search-result page (Mistral 7B, 4096).
 *   q:    [B, hq, S, d] bf16 device;  k, v: [B, hkv, S, d];  out like q
 *   hq % hkv == 0, query head h reads KV head h / (hq/hkv);
 *   S % 128 == 0, d in {64,128}, window >= 1, causal must be 1.
 * Blocks of 128 keys fully outside the band are skipped, fully inside are
 * dense, and only the blocks cut by the band edges are masked per element.
 */
sta_status sta_swa_forward(const void* q, const void* k, const void* v,
                           void* out, int B, int hq, int hkv, int d, int S,
                           int window, int causal, void* stream);

/*
 * sta_swa3d_forward - token-level 3-D sliding-window attention, the
 * mixed-block baseline that README "Why is STA Fast?" compares STA with
 * (token-level windows leave many partially masked blocks).  Every
 * video query token attends to the keys of a window of
 * window_tokens = (Wt, Wh, Ww) TOKENS centred on it and shifted inward at the
 * grid border (clipped to the grid), plus the first text_len text keys; text
 * queries attend to every video key and the first text_len text keys.
 *   q, k, v, out: [B, heads, S, d] bf16 device, RASTER order (as
 *   sta_forward_raster); one window for all heads (HOST int32[3]).
 * The key tiles of a query tile are those holding any key of its tokens'
 * windows; every video block is masked per element.  Requires tiles with
 * ch = cw = 8 and ct even, d in {64,128}, else STA_ERR_UNSUPPORTED.
 */
sta_status sta_swa3d_forward(const void* q, const void* k, const void* v,
                             void* out, int B, int heads, int d, int T, int H,
                             int W, const int tile[3],
                             const int window_tokens[3], int text_len,
                             int has_text, void* stream);

/*
 * Hilbert-order 2-D local attention ("Hilbert-guided block-sparse local
 * attention" blog page): image tokens of an n x n grid (n a power of two,
 * 16 <= n <= 32768) are reordered along a Hilbert curve so that 2-D windows
 * become contiguous runs; block-sparse slide attention then skips more
 * (empty) blocks and masks fewer (partial) ones than in row-by-row order.
 * Curve: recursive quadrant rotation, starting at (0,0), ending at (n-1,0).
 * Slide window: w x w tokens centred on the query, shifted inward at the
 * border.  order: 0 raster (y*n + x; needs n >= 128 so that 128-token blocks
 * are row pieces), 1 Hilbert.
 *
 * sta_hilbert_reorder - [B, heads, n*n, d] bf16 rows, raster -> Hilbert order
 * (to_hilbert = 1: out[pos] = in[raster(pos)]) or back (0).  Bit-exact.
 */
sta_status sta_hilbert_reorder(const void* in, void* out, int B, int heads,
                               int d, int n, int to_hilbert, void* stream);

/*
 * sta_build_slide_block_lists - for each 128-token query block (in `order`),
 * the ascending key blocks holding at least one allowed key, and their class
 * (1 partial, 2 full: every pair of the block allowed), exact; unused slots
 * -1 / 0.  counts: device int32 [nb], ids / classes: device int32
 * [nb][max_k], nb = n*n/128, max_k >= nb (classes may be NULL).
 */
sta_status sta_build_slide_block_lists(int* counts, int* ids, int* classes,
                                       int max_k, int n, int window, int order,
                                       void* stream);

/*
 * sta_slide2d_forward - block-sparse slide attention on q, k, v, out
 * [B, heads, n*n, d] bf16 stored in `order`; each pair of consecutive query
 * blocks runs over the union of their key blocks with a per-element window
 * mask (every non-empty block is treated as partial).  d in {64,128}.
 */
sta_status sta_slide2d_forward(const void* q, const void* k, const void* v,
                               void* out, int B, int heads, int d, int n,
                               int window, int order, void* stream);

/* Synchronises `stream`, returns STA_ERR_DEVICE_BOUNDS if a kernel of the
 * debug build recorded a failed bounds check, else STA_ERR_DEVICE_TIMEOUT if
 * any kernel of this library recorded a gave-up wait since the last call (and
 * clears the record), else STA_ERR_CUDA on a pending CUDA error, else STA_OK. */
sta_status sta_device_status(void* stream);

/*
 * sta_debug_checks - 1 in the debug build of the library (libsta_debug.so,
 * compiled with STA_DEBUG=1), 0 in the release build (libsta.so).  No
 * passage of the pages corresponds to it.  The debug build checks, on the
 * device, that every work item, key-block list entry, TMA row coordinate
 * and output / gradient row lies inside the arrays it indexes; a failed
 * check records STA_ERR_DEVICE_BOUNDS for sta_device_status() and skips the
 * access (nothing traps).  Same entry points, arguments and results.
 */
int sta_debug_checks(void);

/*
 * sta_debug_inject - fault injection for tests; no passage of the pages
 * corresponds to it.  mode 1: the attention kernel's TMA producer skips the
 * Q load, so the MMA warp waits for an arrival that never comes; the bounded
 * wait gives up after wait_limit_ms, the kernel drains its in-flight copies,
 * frees its tensor memory and exits, and sta_device_status() reports
 * STA_ERR_DEVICE_TIMEOUT.  mode 0 with wait_limit_ms = 2000 restores normal
 * operation.  Synchronises the current device; applies to every later launch
 * on it.  No GPU fault, trap or hang is involved.
 */
sta_status sta_debug_inject(int mode, int wait_limit_ms);

/*
 * sta_debug_pair_kernel - kernel selection hook with no counterpart on the
 * pages, for the d = 128 STA forward (sta_forward, sta_forward_lse,
 * sta_forward_raster and the host-buffer form).  pair = 0 (the default): the
 * one-SM kernel that d = 64 and the other modes use; pair = 1: a persistent
 * cluster of two CTAs per pair of SMs, tcgen05 MMAs issued for both SMs at
 * once (M = 256), each SM loading half of every key / value block, three
 * score buffers in tensor memory.  Both compute the same function; the tests
 * run both.  Host-side setting for the calling process; STA_ERR_INVALID_ARG
 * for other values.
 */
sta_status sta_debug_pair_kernel(int pair);

/* Static, never NULL. */
const char* sta_status_string(sta_status s);

/* Releases the per-device workspaces and cached plans. */
void sta_shutdown(void);

/* Effective work of sta_forward: allowed (query, key) pairs over all
 * B*heads, counted on the host from the geometry (FLOPs = 4 * d * pairs). */
int64_t sta_retained_pairs(int B, int heads, int T, int H, int W,
                           const int tile[3], const int* window, int text_len,
                           int has_text);

/* Size of the fixed scratch array used by sta_forward_noalloc (4 MiB). */
#define STA_NOALLOC_SCRATCH_BYTES (4u << 20)

/*
 * sta_forward_noalloc - sta_forward that never allocates memory.  No passage
 * of the STA pages corresponds to it: it exists for callers that cannot let
 * a library call cudaMalloc, e.g. a serving runtime whose memory pool owns
 * the whole device (a stray cudaMalloc can fail or fragment it) or a
 * latency-bound loop that cannot take the implicit device synchronisation of
 * cudaMalloc / cudaFree.
 *
 * Same arguments, layout and numerics as sta_forward; it always runs the
 * one-SM attention kernel (the CTA-pair kernel that sta_debug_pair_kernel(1)
 * selects for sta_forward is never used here), so its output equals
 * sta_forward's with the default kernel bit for bit.  The scratch that
 * sta_forward keeps in its lazily grown workspace (KV tile lists and the work
 * plan) lives instead in one file-scope device array of
 * STA_NOALLOC_SCRATCH_BYTES, which every GPU that loads libsta.so holds until
 * the process exits.
 *
 * Errors: those of sta_forward, plus STA_ERR_SCRATCH_LIMIT when the
 * problem's tile lists and plan do not fit the array (the video+text
 * workload of 115,456 tokens x 24 heads needs about 0.55 MiB).  That size
 * check runs on the host after the argument checks and before the device is
 * queried, so a problem too large for the array gets STA_ERR_SCRATCH_LIMIT
 * even where sta_forward would answer STA_ERR_UNSUPPORTED for the device.
 * Nothing is enqueued on any error.
 *
 * The first call on a device looks up that device's address of the array
 * (cudaGetSymbolAddress, with the device current), so make the first call on
 * each device outside any stream capture.  All calls share the one array and
 * it keeps the last call's contents.  The work plan is copied into it from
 * host memory only when the problem differs from the previous call's; the
 * tile lists are rebuilt by a kernel on every call, so nothing needs
 * clearing.  Calls that overlap on the GPU (different streams, or several
 * host threads) race on the array: order them on one stream.
 * It calls no cudaMalloc, cudaFree or other allocating routine.
 */
sta_status sta_forward_noalloc(const void* q, const void* k, const void* v,
                               void* out, int B, int heads, int d, int T,
                               int H, int W, const int tile[3],
                               const int* window, int text_len, int has_text,
                               void* stream);

#ifdef __cplusplus
}
#endif

#endif /* STA_H_ */
