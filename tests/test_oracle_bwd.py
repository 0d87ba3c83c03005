"""Pins of the STA backward oracle: torch autograd in float64 on the masked
attention, central finite differences, and the row-wise forms."""
import numpy as np
import pytest
import torch

from oracle import sta_bwd_oracle, sta_oracle


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


@pytest.mark.parametrize("case", [
    (4, 4, 6, (2, 2, 2), (1, 2, 3), 0, False),
    (4, 4, 6, (2, 2, 2), (2, 1, 2), 37, True),
    (2, 6, 8, (1, 2, 2), (1, 3, 3), 256, True),
])
def test_matches_autograd(case):
    T, H, W, tile, window, text_len, has_text = case
    S = T * H * W + (256 if has_text else 0)
    q, k, v, do = (_rand((S, 8), s) for s in (1, 2, 3, 4))
    dq, dk, dv, out, _ = sta_bwd_oracle.sta_backward_dense(q, k, v, do, T, H, W, tile, window,
                                                           text_len, has_text)
    mask = torch.from_numpy(sta_oracle.sta_mask(T, H, W, tile, window, text_len, has_text))
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    s = (tq @ tk.T) / np.sqrt(8)
    s = s.masked_fill(~mask, float("-inf"))
    o = torch.softmax(s, dim=1) @ tv
    o.backward(torch.from_numpy(do))
    np.testing.assert_allclose(out, o.detach().numpy(), atol=1e-12)
    np.testing.assert_allclose(dq, tq.grad.numpy(), atol=1e-10)
    np.testing.assert_allclose(dk, tk.grad.numpy(), atol=1e-10)
    np.testing.assert_allclose(dv, tv.grad.numpy(), atol=1e-10)
    if has_text and text_len < 256:       # padded text keys get no gradient
        Lv = T * H * W
        assert np.abs(dk[Lv + text_len:]).max() == 0 and np.abs(dv[Lv + text_len:]).max() == 0


def test_finite_differences():
    T, H, W, tile, window = 2, 2, 4, (1, 2, 2), (1, 1, 1)
    S = T * H * W
    q, k, v, do = (_rand((S, 4), s) for s in (5, 6, 7, 8))
    dq, dk, dv, _, _ = sta_bwd_oracle.sta_backward_dense(q, k, v, do, T, H, W, tile, window, 0,
                                                         False)

    def loss(qq, kk, vv):
        out, _ = sta_oracle.sta_forward_dense(qq, kk, vv, T, H, W, tile, window, 0, False)
        return (out * do).sum()

    eps = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for (i, c) in [(0, 0), (3, 2), (S - 1, 3)]:
            xp, xm = x.copy(), x.copy()
            xp[i, c] += eps
            xm[i, c] -= eps
            args_p = {"qq": q, "kk": k, "vv": v}
            args_m = dict(args_p)
            args_p[name * 2], args_m[name * 2] = xp, xm
            fd = (loss(**args_p) - loss(**args_m)) / (2 * eps)
            assert abs(fd - g[i, c]) < 1e-6, (name, i, c, fd, g[i, c])


def test_row_forms_match_dense():
    T, H, W, tile, window, text_len = 4, 4, 6, (2, 2, 2), (2, 1, 2), 37
    S = T * H * W + 256
    q, k, v, do = (_rand((S, 8), s) for s in (9, 10, 11, 12))
    dq, dk, dv, _, _ = sta_bwd_oracle.sta_backward_dense(q, k, v, do, T, H, W, tile, window,
                                                         text_len, True)
    rows = np.array([0, 7, 50, 95, 96, 200, S - 1])
    np.testing.assert_allclose(sta_bwd_oracle.sta_backward_query_rows(
        q, k, v, do, rows, T, H, W, tile, window, text_len, True), dq[rows], atol=1e-12)
    keys = np.array([0, 13, 95, 96, 96 + 36, 96 + 37, S - 1])
    gk, gv = sta_bwd_oracle.sta_backward_key_rows(q, k, v, do, keys, T, H, W, tile, window,
                                                  text_len, True)
    np.testing.assert_allclose(gk, dk[keys], atol=1e-12)
    np.testing.assert_allclose(gv, dv[keys], atol=1e-12)
    assert not gk[-1].any() and not gv[-1].any()      # padded text key: no gradient
    # without text, border and interior key tiles, every key row
    S = T * H * W
    q, k, v, do = (x[:S] for x in (q, k, v, do))
    _, dk, dv, _, _ = sta_bwd_oracle.sta_backward_dense(q, k, v, do, T, H, W, tile, window, 0,
                                                        False)
    keys = np.arange(S)
    gk, gv = sta_bwd_oracle.sta_backward_key_rows(q, k, v, do, keys, T, H, W, tile, window, 0,
                                                  False)
    np.testing.assert_allclose(gk, dk, atol=1e-12)
    np.testing.assert_allclose(gv, dv, atol=1e-12)
