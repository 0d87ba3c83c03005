"""GPU parity of the forward's rare softmax paths, against the float64 oracle.

The kernels keep a running row maximum and raise it only when a key block's
maximum exceeds it by more than 2^8 (lazy rescale); after the first block a
row then recomputes that block's exponentials against the new maximum and
rescales O and the row sum.  Unit-variance inputs almost never take that
path, so these cases scale chosen keys up:
  * the text keys (the last blocks of every query's key sequence) by 6: the
    maximum rises in the last blocks;
  * the text keys by 40: jumps far above 2^64, where the first exponentials
    against the old maximum overflow and must be discarded;
  * one video tile in the middle of the grid by 4: the maximum rises in the
    middle of the key sequence of the query tiles whose window holds it.
Checked for the one-SM kernel (d = 64 and 128) and the CTA-pair kernel.

Tolerance, from the arithmetic: P enters the P.V product rounded to bf16
(relative error <= 2^-9 per term, so at most 2^-9 max|v| on an output; with
the lazy rescale the dominant term of a peaked row is not exactly 1 and takes
that rounding), and the output itself is stored in bf16 (half an ulp,
<= 2^-8 |o|).  Peaked rows here have |o| up to ~5, so the bound is
elementwise: |err| <= 2^-9 max|v| + 2^-8 |ref| + 1e-3; mean-abs <= 2e-3 per
(b, h); log-sum-exp within 1e-2.
"""
import numpy as np
import pytest
import torch

import block_sparse_local_b200 as sta
from block_sparse_local_b200 import workloads
from oracle import sta_oracle

pytestmark = pytest.mark.gpu

MEAN_ABS = 2e-3
SHAPE, TILE = (12, 16, 24), (6, 8, 8)


@pytest.fixture(autouse=True)
def _needs_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    yield
    sta.use_pair_kernel(False)


def _scaled_keys(w, k, where, factor):
    k = k.clone()
    if where == "text":
        sl = slice(w.L_v, w.L_v + w.text_len)
    else:
        # the tile at the centre of the tile grid, in raster order: a box
        nt, nh, nw = (SHAPE[a] // TILE[a] for a in range(3))
        ct, ch, cw = nt // 2, nh // 2, nw // 2
        idx = []
        for t in range(ct * TILE[0], (ct + 1) * TILE[0]):
            for h in range(ch * TILE[1], (ch + 1) * TILE[1]):
                base = (t * SHAPE[1] + h) * SHAPE[2]
                idx.extend(range(base + cw * TILE[2], base + (cw + 1) * TILE[2]))
        sl = torch.tensor(idx)
    k[:, :, sl, :] = (k[:, :, sl, :].float() * factor).to(torch.bfloat16)
    return k


CASES = [("text", 6.0), ("text", 40.0), ("video", 4.0)]


@pytest.mark.parametrize("where,factor", CASES, ids=lambda x: str(x))
@pytest.mark.parametrize("kernel", ["one_sm_d64", "one_sm_d128", "pair_d128"])
def test_rising_row_max_matches_oracle(where, factor, kernel):
    d = 64 if kernel.endswith("d64") else 128
    windows = [(2, 2, 2), (1, 2, 3)]
    w = workloads.small_sta_case(*SHAPE, TILE, windows, 200, True, d=d, B=1, seed=41)
    q, k, v = workloads.sta_inputs(w)
    k = _scaled_keys(w, k, where, factor)
    sta.use_pair_kernel(kernel.startswith("pair"))
    out, lse = sta.forward_raster(q.cuda(), k.cuda(), v.cuda(), w.windows, w.text_len,
                                  w.has_text, SHAPE, w.tile, return_lse=True)
    sta.device_status()
    got, got_lse = out.float().cpu().numpy(), lse.cpu().numpy()
    q64, k64, v64 = (x.double().numpy() for x in (q, k, v))
    res = sta_oracle.sta_forward_batched(q64, k64, v64, w.T, w.H, w.W, w.tile, w.windows,
                                         w.text_len, w.has_text)
    assert np.isfinite(got).all() and np.isfinite(got_lse).all()
    for (b, h), (ref, ref_lse) in res.items():
        err = np.abs(got[b, h] - ref)
        bound = 2.0 ** -9 * np.abs(v64[b, h]).max() + 2.0 ** -8 * np.abs(ref) + 1e-3
        assert (err <= bound).all() and err.mean() <= MEAN_ABS, (b, h, (err / bound).max(),
                                                                  err.mean())
        assert np.abs(got_lse[b, h] - ref_lse).max() < 1e-2
