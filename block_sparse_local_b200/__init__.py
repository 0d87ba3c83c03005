"""Sliding Tile Attention (STA) forward for NVIDIA B200 (sm_100a).

A thin ctypes binding over libsta.so (include/sta.h).  PyTorch only provides
device memory and the current CUDA stream; every step runs in the library's
CUDA kernels.  There is no CPU fallback: if libsta.so is missing, or the
device is not sm_100, calls raise.

Method (STA README "Sliding Tile Atteniton Kernel", section Usage):
``sliding_tile_attention(q, k, v, window_size, text_length, has_text)`` on
[batch, heads, seq, head_dim] tensors, seq = T*H*W (+ 256 padded text
tokens), tiles of (6, 8, 8) tokens, ``window_size`` in tiles.
"""
import ctypes
import functools
import os

import torch

from .build import DEBUG_LIB_PATH, LIB_PATH

__all__ = [
    "StaError", "lib", "tile_reorder", "tile_unreorder", "build_kv_tile_lists",
    "forward", "sliding_tile_attention", "swa_forward", "device_status",
    "retained_pairs", "STATUS", "forward_noalloc", "forward_raster", "swa3d_forward",
    "hilbert_reorder", "build_slide_block_lists", "slide2d_forward", "slide_attention_2d",
    "backward", "SlidingTileAttentionFunction", "TileReorderFunction",
    "sliding_tile_attention_host", "use_pair_kernel",
]

STATUS = {0: "STA_OK", 1: "STA_ERR_INVALID_ARG", 2: "STA_ERR_UNSUPPORTED",
          3: "STA_ERR_CUDA", 4: "STA_ERR_DEVICE_TIMEOUT", 5: "STA_ERR_SCRATCH_LIMIT",
          6: "STA_ERR_DEVICE_BOUNDS"}

EXPORTED = ("sta_tile_reorder", "sta_tile_unreorder", "sta_build_kv_tile_lists",
            "sta_forward", "sta_forward_lse", "sta_swa_forward",
            "sta_device_status", "sta_status_string", "sta_shutdown",
            "sta_retained_pairs", "sta_forward_noalloc", "sta_forward_raster",
            "sta_swa3d_forward", "sta_debug_inject", "sta_hilbert_reorder",
            "sta_build_slide_block_lists", "sta_slide2d_forward", "sta_backward",
            "sta_forward_raster_host", "sta_debug_pair_kernel", "sta_debug_checks")


class StaError(RuntimeError):
    def __init__(self, code, where):
        self.code = code
        super().__init__(f"{where}: {STATUS.get(code, code)}")


_LIB = None
_DEBUG_LIB = None
_P = ctypes.c_void_p
_I = ctypes.c_int
_I3 = ctypes.c_int * 3


def lib():
    """Loads libsta.so (built in-tree); raises if it is missing."""
    global _LIB
    if _LIB is None:
        _LIB = _load(LIB_PATH)
    return _LIB


def debug_lib():
    """Loads libsta_debug.so, the build with device bounds checks (same entry
    points; a failed check is reported by sta_device_status as
    STA_ERR_DEVICE_BOUNDS); raises if it is missing."""
    global _DEBUG_LIB
    if _DEBUG_LIB is None:
        _DEBUG_LIB = _load(DEBUG_LIB_PATH)
    return _DEBUG_LIB


def _load(path):
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build it with "
            "`python -m block_sparse_local_b200.build`")
    L = ctypes.CDLL(path)
    geo = [_I, _I, _I, _I, _I, _I, ctypes.POINTER(ctypes.c_int)]
    L.sta_tile_reorder.argtypes = [_P, _P] + geo + [_I, _P]
    L.sta_tile_unreorder.argtypes = [_P, _P] + geo + [_I, _P]
    L.sta_build_kv_tile_lists.argtypes = [_P, _P, _I, _I, _I, _I, _I,
                                          ctypes.POINTER(ctypes.c_int),
                                          ctypes.POINTER(ctypes.c_int), _I, _I, _P]
    fwd = [_I, _I, _I, _I, _I, _I, ctypes.POINTER(ctypes.c_int),
           ctypes.POINTER(ctypes.c_int), _I, _I, _P]
    L.sta_forward.argtypes = [_P, _P, _P, _P] + fwd
    L.sta_forward_lse.argtypes = [_P, _P, _P, _P, _P] + fwd
    L.sta_forward_noalloc.argtypes = [_P, _P, _P, _P] + fwd
    L.sta_forward_raster.argtypes = [_P, _P, _P, _P, _P] + fwd
    L.sta_swa3d_forward.argtypes = [_P, _P, _P, _P] + fwd
    L.sta_forward_raster_host.argtypes = [_P, _P, _P, _P] + fwd[:-1] + [ctypes.c_size_t, _P]
    L.sta_swa_forward.argtypes = [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P]
    L.sta_device_status.argtypes = [_P]
    L.sta_debug_inject.argtypes = [_I, _I]
    L.sta_debug_pair_kernel.argtypes = [_I]
    L.sta_backward.argtypes = [_P] * 9 + fwd
    L.sta_hilbert_reorder.argtypes = [_P, _P, _I, _I, _I, _I, _I, _P]
    L.sta_build_slide_block_lists.argtypes = [_P, _P, _P, _I, _I, _I, _I, _P]
    L.sta_slide2d_forward.argtypes = [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P]
    L.sta_status_string.argtypes = [_I]
    L.sta_status_string.restype = ctypes.c_char_p
    L.sta_shutdown.argtypes = []
    L.sta_shutdown.restype = None
    L.sta_retained_pairs.argtypes = [_I, _I, _I, _I, _I, ctypes.POINTER(ctypes.c_int),
                                     ctypes.POINTER(ctypes.c_int), _I, _I]
    L.sta_retained_pairs.restype = ctypes.c_int64
    L.sta_debug_checks.argtypes = []
    for name in EXPORTED:
        fn = getattr(L, name)
        if name not in ("sta_status_string", "sta_shutdown", "sta_retained_pairs"):
            fn.restype = ctypes.c_int
    return L


def _ranged(fn):
    """NVTX range "sta.<name>" around a public call, so that a profiler's
    timeline shows which library call launched which kernels."""
    name = "sta." + fn.__name__

    @functools.wraps(fn)
    def wrapper(*args, **kwargs):
        torch.cuda.nvtx.range_push(name)
        try:
            return fn(*args, **kwargs)
        finally:
            torch.cuda.nvtx.range_pop()
    return wrapper


def _check(code, where):
    if code != 0:
        raise StaError(code, where)


def _stream(t):
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _windows(window_size, heads):
    ws = [tuple(int(x) for x in w) for w in window_size]
    if len(ws) == 1 and heads > 1:
        ws = ws * heads
    if len(ws) != heads:
        raise ValueError("window_size needs one (wt, wh, ww) per head (or one for all)")
    arr = (ctypes.c_int * (3 * heads))(*[x for w in ws for x in w])
    return arr


def _check_qkv(*ts):
    for t in ts:
        if not t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError("tensors must be contiguous bf16 CUDA tensors")


@_ranged
def tile_reorder(x, video_shape, tile=(6, 8, 8), has_text=True, out=None):
    """[B, heads, S, d] raster order -> tile order (text rows unchanged)."""
    _check_qkv(x)
    out = torch.empty_like(x) if out is None else out
    B, nh, _, d = x.shape
    T, H, W = video_shape
    _check(lib().sta_tile_reorder(_ptr(x), _ptr(out), B, nh, d, T, H, W, _I3(*tile),
                                  int(has_text), _stream(x)), "sta_tile_reorder")
    return out


@_ranged
def tile_unreorder(x, video_shape, tile=(6, 8, 8), has_text=True, out=None):
    """Inverse of tile_reorder."""
    _check_qkv(x)
    out = torch.empty_like(x) if out is None else out
    B, nh, _, d = x.shape
    T, H, W = video_shape
    _check(lib().sta_tile_unreorder(_ptr(x), _ptr(out), B, nh, d, T, H, W, _I3(*tile),
                                    int(has_text), _stream(x)), "sta_tile_unreorder")
    return out


@_ranged
def build_kv_tile_lists(window_size, video_shape, tile=(6, 8, 8), text_length=0,
                        has_text=True, max_k=None, device="cuda"):
    """Per-head KV tile lists: (counts [heads, NQ], ids [heads, NQ, max_k])."""
    heads = len(window_size)
    T, H, W = video_shape
    NV = (T // tile[0]) * (H // tile[1]) * (W // tile[2])
    NQ = NV + (1 if has_text else 0)
    if max_k is None:
        max_k = NV + 1
    counts = torch.empty((heads, NQ), dtype=torch.int32, device=device)
    ids = torch.empty((heads, NQ, max_k), dtype=torch.int32, device=device)
    _check(lib().sta_build_kv_tile_lists(_ptr(counts), _ptr(ids), max_k, heads, T, H, W,
                                         _I3(*tile), _windows(window_size, heads),
                                         int(text_length), int(has_text), _stream(counts)),
           "sta_build_kv_tile_lists")
    return counts, ids


@_ranged
def forward(q, k, v, window_size, text_length, has_text, video_shape,
            tile=(6, 8, 8), out=None, return_lse=False):
    """STA attention on TILE-ordered q, k, v [B, heads, S, d] (bf16)."""
    _check_qkv(q, k, v)
    B, nh, S, d = q.shape
    T, H, W = video_shape
    out = torch.empty_like(q) if out is None else out
    wins = _windows(window_size, nh)
    if return_lse:
        lse = torch.empty((B, nh, S), dtype=torch.float32, device=q.device)
        _check(lib().sta_forward_lse(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B,
                                     nh, d, T, H, W, _I3(*tile), wins, int(text_length),
                                     int(has_text), _stream(q)), "sta_forward_lse")
        return out, lse
    _check(lib().sta_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, nh, d, T, H, W,
                             _I3(*tile), wins, int(text_length), int(has_text),
                             _stream(q)), "sta_forward")
    return out


@_ranged
def forward_noalloc(q, k, v, window_size, text_length, has_text, video_shape,
                    tile=(6, 8, 8), out=None):
    """Like forward(), through sta_forward_noalloc: the library allocates no
    device memory (its scratch is a fixed 4 MiB array); for callers whose
    memory pool owns the device or that cannot take cudaMalloc's implicit
    synchronisation.  Calls that overlap on the GPU race on the shared array."""
    _check_qkv(q, k, v)
    B, nh, S, d = q.shape
    T, H, W = video_shape
    out = torch.empty_like(q) if out is None else out
    _check(lib().sta_forward_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, nh, d, T, H, W,
                                     _I3(*tile), _windows(window_size, nh), int(text_length),
                                     int(has_text), _stream(q)), "sta_forward_noalloc")
    return out


@_ranged
def forward_raster(q, k, v, window_size, text_length, has_text, video_shape,
                   tile=(6, 8, 8), out=None, return_lse=False):
    """STA attention on RASTER-ordered q, k, v with the permutation fused into
    the kernel (sta_forward_raster).  Raises StaError(STA_ERR_UNSUPPORTED) when
    a 128-row block of a tile is not a box of the grid."""
    _check_qkv(q, k, v)
    B, nh, S, d = q.shape
    T, H, W = video_shape
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, nh, S), dtype=torch.float32, device=q.device) if return_lse else None
    _check(lib().sta_forward_raster(_ptr(q), _ptr(k), _ptr(v), _ptr(out),
                                    None if lse is None else _ptr(lse), B, nh, d, T, H, W,
                                    _I3(*tile), _windows(window_size, nh), int(text_length),
                                    int(has_text), _stream(q)), "sta_forward_raster")
    return (out, lse) if return_lse else out


@_ranged
def backward(q, k, v, out, dout, lse, window_size, text_length, has_text, video_shape,
             tile=(6, 8, 8)):
    """Gradients (dq, dk, dv) of forward() on TILE-ordered tensors; lse from
    forward(..., return_lse=True)."""
    _check_qkv(q, k, v, out, dout)
    B, nh, S, d = q.shape
    T, H, W = video_shape
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    _check(lib().sta_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse),
                              _ptr(dq), _ptr(dk), _ptr(dv), B, nh, d, T, H, W, _I3(*tile),
                              _windows(window_size, nh), int(text_length), int(has_text),
                              _stream(q)), "sta_backward")
    return dq, dk, dv


class SlidingTileAttentionFunction(torch.autograd.Function):
    """Differentiable STA on TILE-ordered q, k, v (forward keeps the LSE)."""

    @staticmethod
    def forward(ctx, q, k, v, window_size, text_length, has_text, video_shape, tile):
        out, lse = forward(q, k, v, window_size, text_length, has_text, video_shape, tile,
                           return_lse=True)
        ctx.save_for_backward(q, k, v, out, lse)
        ctx.args = (window_size, text_length, has_text, video_shape, tile)
        return out

    @staticmethod
    def backward(ctx, dout):
        q, k, v, out, lse = ctx.saved_tensors
        dq, dk, dv = backward(q, k, v, out, dout.contiguous(), lse, *ctx.args)
        return dq, dk, dv, None, None, None, None, None


class TileReorderFunction(torch.autograd.Function):
    """Differentiable raster -> tile permutation (its gradient is the inverse)."""

    @staticmethod
    def forward(ctx, x, video_shape, tile, has_text, to_tile):
        ctx.args = (video_shape, tile, has_text, to_tile)
        f = tile_reorder if to_tile else tile_unreorder
        return f(x.contiguous(), video_shape, tile, has_text)

    @staticmethod
    def backward(ctx, g):
        video_shape, tile, has_text, to_tile = ctx.args
        f = tile_unreorder if to_tile else tile_reorder
        return f(g.contiguous(), video_shape, tile, has_text), None, None, None, None


@_ranged
def sliding_tile_attention(q, k, v, window_size, text_length, has_text=True,
                           video_shape=(30, 48, 80), tile=(6, 8, 8), fused=True):
    """README-style call on RASTER-ordered q, k, v.

    fused=True: one attention kernel reads and writes raster order directly
    (sta_forward_raster); tile shapes whose blocks are not boxes of the grid
    go through the explicit reorder -> attend -> unreorder kernels instead.
    When an input requires grad, the call is differentiable (permutation,
    attention with saved log-sum-exp, inverse permutation; backward by
    sta_backward).
    """
    if torch.is_grad_enabled() and any(t.requires_grad for t in (q, k, v)):
        qt, kt, vt = (TileReorderFunction.apply(x, video_shape, tile, has_text, True)
                      for x in (q, k, v))
        ot = SlidingTileAttentionFunction.apply(qt, kt, vt, window_size, text_length,
                                                has_text, video_shape, tile)
        return TileReorderFunction.apply(ot, video_shape, tile, has_text, False)
    if fused:
        try:
            return forward_raster(q, k, v, window_size, text_length, has_text, video_shape,
                                  tile)
        except StaError as e:
            if e.code != 2:
                raise
    qt = tile_reorder(q, video_shape, tile, has_text)
    kt = tile_reorder(k, video_shape, tile, has_text)
    vt = tile_reorder(v, video_shape, tile, has_text)
    ot = forward(qt, kt, vt, window_size, text_length, has_text, video_shape, tile)
    return tile_unreorder(ot, video_shape, tile, has_text)


@_ranged
def sliding_tile_attention_host(q, k, v, window_size, text_length, has_text=True,
                                video_shape=(30, 48, 80), tile=(6, 8, 8), out=None,
                                device=None, blocking=True, chunk_bytes=0):
    """The README call on HOST tensors (sta_forward_raster_host).

    q, k, v: CPU bf16 [B, heads, S, d], raster order, contiguous; pin them
    (``tensor.pin_memory()``) so the copies overlap the attention.  The
    library streams whole heads through device staging buffers on
    ``device`` (default: the current CUDA device), at most ``chunk_bytes``
    per tensor and chunk (0: the library default), and writes ``out``, a CPU
    tensor (pinned when allocated here).  With blocking=False the call only
    enqueues the work on the device's current stream: synchronise that stream
    before reading ``out`` or touching q, k, v.
    """
    for t in (q, k, v):
        if t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError("tensors must be contiguous bf16 CPU tensors")
    if not (q.shape == k.shape == v.shape):
        raise ValueError("q, k, v must have one shape")
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None \
        else torch.device(device)
    if out is None:
        out = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
    elif out.is_cuda or out.shape != q.shape or out.dtype != q.dtype or \
            not out.is_contiguous():
        raise ValueError("out must be a contiguous bf16 CPU tensor shaped like q")
    B, nh, S, d = q.shape
    T, H, W = video_shape
    with torch.cuda.device(dev):
        stream = torch.cuda.current_stream(dev)
        _check(lib().sta_forward_raster_host(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, nh, d,
                                             T, H, W, _I3(*tile), _windows(window_size, nh),
                                             int(text_length), int(has_text),
                                             int(chunk_bytes),
                                             ctypes.c_void_p(stream.cuda_stream)),
               "sta_forward_raster_host")
        if blocking:
            stream.synchronize()
    return out


@_ranged
def swa3d_forward(q, k, v, window_tokens, text_length, has_text, video_shape,
                  tile=(6, 8, 8), out=None):
    """Token-level 3-D sliding-window attention on RASTER-ordered q, k, v:
    each query sees a window of (Wt, Wh, Ww) tokens around it (the mixed-block
    baseline of STA); tiles must have 8 x 8 tokens per t-slice."""
    _check_qkv(q, k, v)
    B, nh, S, d = q.shape
    T, H, W = video_shape
    out = torch.empty_like(q) if out is None else out
    _check(lib().sta_swa3d_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, nh, d, T, H, W,
                                   _I3(*tile), _I3(*window_tokens), int(text_length),
                                   int(has_text), _stream(q)), "sta_swa3d_forward")
    return out


ORDERS = {"raster": 0, "hilbert": 1}


@_ranged
def hilbert_reorder(x, n, to_hilbert=True, out=None):
    """[B, heads, n*n, d] rows between raster and Hilbert order (bit-exact)."""
    _check_qkv(x)
    out = torch.empty_like(x) if out is None else out
    B, nh, _, d = x.shape
    _check(lib().sta_hilbert_reorder(_ptr(x), _ptr(out), B, nh, d, n, int(to_hilbert),
                                     _stream(x)), "sta_hilbert_reorder")
    return out


@_ranged
def build_slide_block_lists(n, window, order="hilbert", device="cuda"):
    """(counts [nb], ids [nb, nb], classes [nb, nb]) of 2-D slide attention."""
    nb = n * n // 128
    counts = torch.empty(nb, dtype=torch.int32, device=device)
    ids = torch.empty((nb, nb), dtype=torch.int32, device=device)
    cls = torch.empty((nb, nb), dtype=torch.int32, device=device)
    _check(lib().sta_build_slide_block_lists(_ptr(counts), _ptr(ids), _ptr(cls), nb, n,
                                             int(window), ORDERS[order], _stream(counts)),
           "sta_build_slide_block_lists")
    return counts, ids, cls


@_ranged
def slide2d_forward(q, k, v, n, window, order="hilbert", out=None):
    """Block-sparse 2-D slide attention on q, k, v stored in `order`."""
    _check_qkv(q, k, v)
    B, nh, _, d = q.shape
    out = torch.empty_like(q) if out is None else out
    _check(lib().sta_slide2d_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, nh, d, n,
                                     int(window), ORDERS[order], _stream(q)),
           "sta_slide2d_forward")
    return out


@_ranged
def slide_attention_2d(q, k, v, n, window, order="hilbert"):
    """Raster-ordered in and out; with order='hilbert' the tokens are reordered
    along the Hilbert curve, attended block-sparsely, and put back."""
    if order == "raster":
        return slide2d_forward(q, k, v, n, window, "raster")
    qh, kh, vh = (hilbert_reorder(x, n, True) for x in (q, k, v))
    oh = slide2d_forward(qh, kh, vh, n, window, "hilbert")
    return hilbert_reorder(oh, n, False)


@_ranged
def swa_forward(q, k, v, window, causal=True, out=None):
    """Token-level causal sliding-window attention, GQA: q [B,hq,S,d], k,v [B,hkv,S,d]."""
    _check_qkv(q, k, v)
    B, hq, S, d = q.shape
    hkv = k.shape[1]
    out = torch.empty_like(q) if out is None else out
    _check(lib().sta_swa_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, hq, hkv, d, S,
                                 int(window), int(bool(causal)), _stream(q)),
           "sta_swa_forward")
    return out


def use_pair_kernel(pair=True):
    """Kernel selection hook for the d = 128 STA forward: CTA pairs
    (pair=True) or the one-SM kernel (pair=False, the library default)."""
    _check(lib().sta_debug_pair_kernel(int(bool(pair))), "sta_debug_pair_kernel")


def device_status(device=None):
    """Synchronises the current stream and reports a gave-up device wait."""
    dev = torch.device("cuda") if device is None else torch.device(device)
    s = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    _check(lib().sta_device_status(s), "sta_device_status")


def retained_pairs(B, window_size, video_shape, tile=(6, 8, 8), text_length=0,
                   has_text=True):
    """Allowed (query, key) pairs of sta_forward (FLOPs = 4 * d * pairs)."""
    heads = len(window_size)
    T, H, W = video_shape
    n = lib().sta_retained_pairs(B, heads, T, H, W, _I3(*tile), _windows(window_size, heads),
                                 int(text_length), int(has_text))
    if n < 0:
        raise ValueError("invalid geometry")
    return int(n)
