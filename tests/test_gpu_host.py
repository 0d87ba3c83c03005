"""GPU parity of sta_forward_raster_host (q, k, v and out in host memory,
streamed through device staging buffers in chunks of whole heads).

The host path runs the same kernels as sta_forward_raster on the same
slices, so its output must equal the device call's bit for bit; the small
case is also checked against the float64 oracle (max-abs <= 2e-2, mean-abs
<= 2e-3 per (batch, head)).  Chunk sizes are forced small so one call walks
several chunks through both staging buffers, with a shorter last chunk.
"""
import numpy as np
import pytest
import torch

import block_sparse_local_b200 as sta
from block_sparse_local_b200 import workloads
from oracle import sta_oracle

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 2e-2, 2e-3


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    sta.lib()


def _device_ref(w, q, k, v):
    o = sta.forward_raster(q.cuda(), k.cuda(), v.cuda(), w.windows, w.text_len, w.has_text,
                           (w.T, w.H, w.W), w.tile)
    sta.device_status()
    return o.cpu()


def _small():
    # 2 x 3 x 4 tiles of (2, 8, 8) tokens, five heads with three windows,
    # two batch elements, 37 valid text keys
    return workloads.small_sta_case(4, 24, 32, (2, 8, 8),
                                    [(1, 3, 3), (2, 2, 4), (1, 3, 3), (2, 3, 1), (1, 1, 1)],
                                    37, True, d=128, B=2, seed=21)


@pytest.mark.parametrize("heads_per_chunk", [1, 2, 5])
def test_host_path_equals_device_path(heads_per_chunk):
    w = _small()
    q, k, v = (x.pin_memory() for x in workloads.sta_inputs(w))
    slice_bytes = w.S * w.d * 2
    out = sta.sliding_tile_attention_host(q, k, v, w.windows, w.text_len, w.has_text,
                                          (w.T, w.H, w.W), w.tile,
                                          chunk_bytes=heads_per_chunk * slice_bytes)
    sta.device_status()
    ref = _device_ref(w, q, k, v)
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    got = out.float().numpy()
    q64, k64, v64 = (x.double().numpy() for x in (q, k, v))
    res = sta_oracle.sta_forward_batched(q64, k64, v64, w.T, w.H, w.W, w.tile, w.windows,
                                         w.text_len, w.has_text)
    for (b, h), (r, _) in res.items():
        err = np.abs(got[b, h] - r)
        assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (b, h, err.max(), err.mean())


def test_host_path_back_to_back_calls_and_pageable_memory():
    # two calls enqueued without a host sync between them reuse the staging
    # buffers; the second must not see the first one's data
    w = _small()
    slice_bytes = w.S * w.d * 2
    q1, k1, v1 = (x.pin_memory() for x in workloads.sta_inputs(w))
    w2 = workloads.small_sta_case(w.T, w.H, w.W, w.tile, w.windows, w.text_len, w.has_text,
                                  d=w.d, B=w.B, seed=22)
    q2, k2, v2 = workloads.sta_inputs(w2)          # pageable
    o1 = sta.sliding_tile_attention_host(q1, k1, v1, w.windows, w.text_len, w.has_text,
                                         (w.T, w.H, w.W), w.tile, blocking=False,
                                         chunk_bytes=2 * slice_bytes)
    o2 = sta.sliding_tile_attention_host(q2, k2, v2, w.windows, w.text_len, w.has_text,
                                         (w.T, w.H, w.W), w.tile, blocking=False,
                                         chunk_bytes=3 * slice_bytes)
    torch.cuda.current_stream().synchronize()
    sta.device_status()
    assert torch.equal(o1.view(torch.int16), _device_ref(w, q1, k1, v1).view(torch.int16))
    assert torch.equal(o2.view(torch.int16), _device_ref(w2, q2, k2, v2).view(torch.int16))


def test_host_path_full_video_text_workload():
    # the benchmarked workload (24 heads, 115,456 rows, d=128) with the
    # default chunking, as bench.py's end-to-end leg runs it
    w = workloads.VIDEO_TEXT
    q, k, v = (x.cpu().pin_memory() for x in workloads.sta_inputs(w, device="cuda"))
    out = sta.sliding_tile_attention_host(q, k, v, w.windows, w.text_len, w.has_text,
                                          (w.T, w.H, w.W), w.tile)
    sta.device_status()
    ref = _device_ref(w, q, k, v)
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
