"""GPU parity of the STA backward pass against the float64 oracle.

Tolerance: gradients scale with the inputs, so errors are measured relative
to the reference: max-abs error <= 2e-2 * max|ref| and mean-abs error
<= 1e-2 * mean|ref| per (batch, head) and tensor (bf16 inputs, P and dS
rounded to bf16 for the MMAs, fp32 accumulation).
"""
import numpy as np
import pytest
import torch

import block_sparse_local_b200 as sta
from block_sparse_local_b200 import workloads
from oracle import perm_oracle, sta_bwd_oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    sta.lib()


def _close(got, ref, what):
    err = np.abs(got - ref)
    assert err.max() <= 2e-2 * np.abs(ref).max(), (what, err.max(), np.abs(ref).max())
    assert err.mean() <= 1e-2 * np.abs(ref).mean(), (what, err.mean(), np.abs(ref).mean())


def _to_tile(x, w):
    return torch.from_numpy(perm_oracle.reorder(x.view(torch.int16).numpy(), w.T, w.H, w.W,
                                                w.tile, w.has_text)).view(torch.bfloat16)


def _from_tile(x, w):
    return perm_oracle.unreorder(x.float().cpu().numpy(), w.T, w.H, w.W, w.tile, w.has_text)


CASES = [
    ((4, 16, 24), (2, 8, 8), [(1, 2, 2)], 0, False, 64),
    ((4, 16, 24), (2, 8, 8), [(2, 1, 3), (1, 2, 1)], 77, True, 128),
    ((6, 8, 16), (6, 8, 8), [(1, 1, 2)], 200, True, 64),
    ((4, 8, 16), (2, 8, 8), [(2, 1, 2)], 256, True, 128),
    ((4, 8, 16), (2, 8, 8), [(1, 1, 1)], 0, True, 64),    # text rows, no valid text key
    # 2 and 3 key blocks per video query block: fewer than the dQ kernel's
    # three K stages, so its rings and drains run partly empty
    ((2, 8, 16), (2, 8, 8), [(1, 1, 1)], 100, True, 128),
    ((2, 8, 16), (2, 8, 8), [(1, 1, 2)], 100, True, 128),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0]}-{c[1]}-t{c[3]}-d{c[5]}")
def test_backward_matches_oracle(case):
    shape, tile, windows, text_len, has_text, d = case
    w = workloads.small_sta_case(*shape, tile, windows, text_len, has_text, d=d, seed=41)
    q, k, v = workloads.sta_inputs(w)
    dout = workloads.randn_bf16(q.shape, 4242)
    qt, kt, vt, dot = (_to_tile(x, w).cuda() for x in (q, k, v, dout))
    out, lse = sta.forward(qt, kt, vt, w.windows, text_len, has_text, shape, tile, return_lse=True)
    dq, dk, dv = sta.backward(qt, kt, vt, out, dot, lse, w.windows, text_len, has_text, shape, tile)
    sta.device_status()
    got = {n: _from_tile(x, w) for n, x in (("dq", dq), ("dk", dk), ("dv", dv))}
    for h in range(w.heads):
        x64 = [x[0, h].double().numpy() for x in (q, k, v, dout)]
        rdq, rdk, rdv, _, _ = sta_bwd_oracle.sta_backward_dense(*x64, *shape, tile, windows[h],
                                                                text_len, has_text)
        _close(got["dq"][0, h], rdq, f"dq h{h}")
        _close(got["dk"][0, h], rdk, f"dk h{h}")
        _close(got["dv"][0, h], rdv, f"dv h{h}")
        if has_text and text_len < 256:
            Lv = w.T * w.H * w.W
            assert np.abs(got["dk"][0, h][Lv + text_len:]).max() == 0
            assert np.abs(got["dv"][0, h][Lv + text_len:]).max() == 0


def test_autograd_function():
    w = workloads.small_sta_case(4, 16, 24, (2, 8, 8), [(1, 2, 2)], 40, True, d=64, seed=43)
    q, k, v = workloads.sta_inputs(w)
    dout = workloads.randn_bf16(q.shape, 4343)
    qt, kt, vt = (_to_tile(x, w).cuda().requires_grad_() for x in (q, k, v))
    out = sta.SlidingTileAttentionFunction.apply(qt, kt, vt, w.windows, w.text_len, True,
                                                 (w.T, w.H, w.W), w.tile)
    out.backward(_to_tile(dout, w).cuda())
    sta.device_status()
    x64 = [x[0, 0].double().numpy() for x in (q, k, v, dout)]
    rdq, rdk, rdv, _, _ = sta_bwd_oracle.sta_backward_dense(*x64, w.T, w.H, w.W, w.tile,
                                                            w.windows[0], w.text_len, True)
    _close(_from_tile(qt.grad, w)[0, 0], rdq, "dq")
    _close(_from_tile(kt.grad, w)[0, 0], rdk, "dk")
    _close(_from_tile(vt.grad, w)[0, 0], rdv, "dv")


def test_backward_full_size_dq_sampled():
    w = workloads.VIDEO_TEXT
    q, k, v = workloads.sta_inputs(w, device="cuda")
    dout = workloads.randn_bf16(q.shape, 4545, device="cuda")
    shape = (w.T, w.H, w.W)
    qt, kt, vt, dot = (sta.tile_reorder(x, shape, w.tile, True) for x in (q, k, v, dout))
    out, lse = sta.forward(qt, kt, vt, w.windows, w.text_len, True, shape, w.tile,
                           return_lse=True)
    dq, dk, dv = sta.backward(qt, kt, vt, out, dot, lse, w.windows, w.text_len, True, shape,
                              w.tile)
    dq = sta.tile_unreorder(dq, shape, w.tile, True)
    sta.device_status()
    rows = np.unique(np.concatenate([np.random.default_rng(7).integers(0, w.L_v, 48),
                                     np.arange(w.L_v, w.L_v + 8)]))
    for h in (0, 17):
        x64 = [x[0, h].double().cpu().numpy() for x in (q, k, v, dout)]
        ref = sta_bwd_oracle.sta_backward_query_rows(*x64, rows, w.T, w.H, w.W, w.tile,
                                                     w.windows[h], w.text_len, True)
        _close(dq[0, h].float().cpu().numpy()[rows], ref, f"dq h{h}")
    for x in (dk, dv):
        assert torch.isfinite(x.float()).all()


def test_raster_api_is_differentiable():
    w = workloads.small_sta_case(4, 16, 24, (2, 8, 8), [(1, 2, 2), (2, 1, 3)], 33, True, d=128,
                                 seed=47)
    q, k, v = workloads.sta_inputs(w)
    dout = workloads.randn_bf16(q.shape, 4747)
    qd, kd, vd = (x.cuda().requires_grad_() for x in (q, k, v))
    out = sta.sliding_tile_attention(qd, kd, vd, w.windows, w.text_len, True, (w.T, w.H, w.W),
                                     w.tile)
    out.backward(dout.cuda())
    sta.device_status()
    for h in range(w.heads):
        x64 = [x[0, h].double().numpy() for x in (q, k, v, dout)]
        rdq, rdk, rdv, rout, _ = sta_bwd_oracle.sta_backward_dense(
            *x64, w.T, w.H, w.W, w.tile, w.windows[h], w.text_len, True)
        _close(out[0, h].detach().float().cpu().numpy(), rout, f"out h{h}")
        _close(qd.grad[0, h].float().cpu().numpy(), rdq, f"dq h{h}")
        _close(kd.grad[0, h].float().cpu().numpy(), rdk, f"dk h{h}")
        _close(vd.grad[0, h].float().cpu().numpy(), rdv, f"dv h{h}")
