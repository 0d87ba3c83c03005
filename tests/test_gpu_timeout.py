"""Failure detection on the GPU without a fault: a missing TMA arrival is
injected (the producer skips the Q load), the bounded device wait gives up,
the kernel unwinds, the host reads STA_ERR_DEVICE_TIMEOUT, and the same
context then computes correct results again."""
import numpy as np
import pytest
import torch

import block_sparse_local_b200 as sta
from block_sparse_local_b200 import workloads
from oracle import sta_oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    sta.lib()


def test_missing_arrival_is_reported_and_context_survives():
    L = sta.lib()
    w = workloads.small_sta_case(12, 16, 24, (6, 8, 8), [(2, 2, 2)], 50, True, d=128, seed=29)
    q, k, v = workloads.sta_inputs(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    shape = (w.T, w.H, w.W)
    assert L.sta_debug_inject(1, 50) == 0
    try:
        sta.forward_raster(qd, kd, vd, w.windows, w.text_len, w.has_text, shape, w.tile)
        with pytest.raises(sta.StaError) as err:
            sta.device_status()
        assert err.value.code == 4            # STA_ERR_DEVICE_TIMEOUT
    finally:
        assert L.sta_debug_inject(0, 2000) == 0
    sta.device_status()                       # the error word was cleared
    out = sta.forward_raster(qd, kd, vd, w.windows, w.text_len, w.has_text, shape, w.tile)
    sta.device_status()
    q64, k64, v64 = (x[0, 0].double().numpy() for x in (q, k, v))
    ref, _ = sta_oracle.sta_forward_rows(q64, k64, v64, w.T, w.H, w.W, w.tile, w.windows[0],
                                         w.text_len, w.has_text)
    err = np.abs(out[0, 0].float().cpu().numpy() - ref)
    assert err.max() <= 2e-2 and err.mean() <= 2e-3
