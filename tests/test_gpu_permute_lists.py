"""GPU parity of the integer paths: token permutation and KV tile lists,
bit-exact against the oracle (through the C ABI)."""
import numpy as np
import pytest
import torch

import block_sparse_local_b200 as sta
from block_sparse_local_b200 import workloads
from oracle import perm_oracle, tiles_oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    sta.lib()   # fails loudly when the library is missing


PERM_CASES = [
    # B, heads, d, (T, H, W), tile, has_text
    (1, 1, 64, (18, 24, 32), (6, 8, 8), False),
    (2, 3, 128, (12, 16, 24), (6, 8, 8), True),
    (1, 2, 64, (1, 64, 48), (1, 16, 16), False),
    (1, 1, 32, (4, 6, 10), (2, 3, 5), True),      # ragged tile sizes
    (1, 1, 256, (2, 4, 4), (1, 2, 2), True),
]


@pytest.mark.parametrize("B,nh,d,shape,tile,has_text", PERM_CASES)
def test_reorder_bit_exact(B, nh, d, shape, tile, has_text):
    T, H, W = shape
    S = T * H * W + (256 if has_text else 0)
    x = torch.randint(-32768, 32767, (B, nh, S, d), dtype=torch.int16).view(torch.bfloat16)
    y = sta.tile_reorder(x.cuda(), shape, tile, has_text)
    want = perm_oracle.reorder(x.view(torch.int16).numpy(), T, H, W, tile, has_text)
    assert np.array_equal(y.cpu().view(torch.int16).numpy(), want)
    z = sta.tile_unreorder(y, shape, tile, has_text)
    assert torch.equal(z.cpu().view(torch.int16), x.view(torch.int16))
    sta.device_status()


def test_reorder_full_size_video_text():
    # every element of two heads carries its own (head, row, column) code, so
    # the whole output is checked against the oracle's index formula
    w = workloads.VIDEO_TEXT
    heads = 2
    row = torch.arange(w.S, dtype=torch.int32, device="cuda")[None, :, None]
    col = torch.arange(w.d, dtype=torch.int32, device="cuda")[None, None, :]
    hd = torch.arange(heads, dtype=torch.int32, device="cuda")[:, None, None]
    code = (row * 131 + col * 7 + hd * 1009) % 65536 - 32768
    xb = code.to(torch.int16)[None].contiguous().view(torch.bfloat16)
    y = sta.tile_reorder(xb, (w.T, w.H, w.W), w.tile, True)
    p = perm_oracle.tile_position_of_raster(w.T, w.H, w.W, w.tile)
    inv = np.empty_like(p)
    inv[p] = np.arange(p.size)
    src = torch.from_numpy(np.concatenate([inv, np.arange(w.L_v, w.S)])).cuda()
    want = xb.view(torch.int16).index_select(2, src)
    assert torch.equal(y.view(torch.int16), want)
    assert torch.equal(sta.tile_unreorder(y, (w.T, w.H, w.W), w.tile, True).view(torch.int16),
                       xb.view(torch.int16))
    sta.device_status()


LIST_CASES = [
    ((18, 24, 32), (6, 8, 8), [(1, 3, 3)], 0, False),              # tiny workload
    ((1, 10, 10), (1, 2, 2), [(1, 3, 3)], 0, False),               # README 2-D demo
    ((30, 48, 80), (6, 8, 8), [(3, 3, 3)] * 2, 200, True),         # video + text
    ((30, 48, 80), (6, 8, 8), [(3, 3, 3)], 0, True),               # no valid text key
    ((36, 48, 48), (6, 8, 8), list(workloads.per_head_windows_video_only()[:6]), 0, False),
    ((1, 256, 256), (1, 16, 16), [(1, 5, 5), (1, 16, 16), (1, 4, 6)], 0, False),
    ((12, 16, 24), (6, 8, 8), [(9, 9, 9), (1, 1, 1), (2, 2, 2)], 256, True),
]


@pytest.mark.parametrize("shape,tile,windows,text_len,has_text", LIST_CASES)
def test_tile_lists_bit_exact(shape, tile, windows, text_len, has_text):
    counts_o, ids_o = tiles_oracle.kv_tile_lists(*shape, tile, windows, text_len, has_text)
    max_k = ids_o.shape[2] + 3
    counts, ids = sta.build_kv_tile_lists(windows, shape, tile, text_len, has_text, max_k=max_k)
    sta.device_status()
    assert np.array_equal(counts.cpu().numpy(), counts_o)
    ids_pad = np.full(ids.shape, -1, dtype=np.int32)
    ids_pad[:, :, :ids_o.shape[2]] = ids_o
    assert np.array_equal(ids.cpu().numpy(), ids_pad)
