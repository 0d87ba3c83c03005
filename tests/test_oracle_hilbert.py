"""Pins of the Hilbert-order oracle: the curve's defining properties and the
block statistics of 2-D slide attention."""
import os

import numpy as np
import pytest

from oracle import hilbert_oracle as ho
from oracle import swa3d_oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_curve_n4_equals_hand_derived_sequence():
    # tests/golden/hilbert_n4.txt: the 16 cells derived by hand from the
    # 2 x 2 curve and the quadrant rotations (a wrong sub-quadrant
    # orientation that stays continuous changes this sequence)
    want = []
    with open(os.path.join(GOLDEN, "hilbert_n4.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                d, x, y = (int(t) for t in line.split())
                assert d == len(want)
                want.append((x, y))
    assert [ho.hilbert_d2xy(4, d) for d in range(16)] == want


@pytest.mark.parametrize("n", [4, 8, 16, 32])
def test_every_level_is_the_curve_of_its_quadrant(n):
    # Recursive structure at every level s: positions [m s^2, (m+1) s^2) fill
    # one aligned s x s square, and the curve inside it, moved to the origin,
    # is the s x s curve itself, one of its two diagonal reflections, or its
    # half turn (the composition of both reflections, which appears from the
    # third level on).
    order = ho.hilbert_order(n)
    xs, ys = order % n, order // n
    s = 2
    while s <= n:
        base = [ho.hilbert_d2xy(s, d) for d in range(s * s)]
        transposed = [(y, x) for x, y in base]
        anti = [(s - 1 - y, s - 1 - x) for x, y in base]
        for m in range(n * n // (s * s)):
            cx, cy = xs[m * s * s:(m + 1) * s * s], ys[m * s * s:(m + 1) * s * s]
            x0, y0 = cx.min(), cy.min()
            assert x0 % s == 0 and y0 % s == 0
            assert cx.max() - x0 == s - 1 and cy.max() - y0 == s - 1
            local = list(zip((cx - x0).tolist(), (cy - y0).tolist()))
            mirrored = [(s - 1 - x, s - 1 - y) for x, y in base]
            assert local in (base, transposed, anti, mirrored), (s, m)
        s *= 2


def test_block_classes_equal_a_plain_loop():
    # every (query, key) pair tested one by one from its (x, y) coordinates,
    # small blocks so that partial, full and empty blocks all occur
    n, w, block = 8, 3, 8
    for order in (ho.raster_order(n), ho.hilbert_order(n)):
        nb = n * n // block
        cnt = np.zeros((nb, nb), dtype=np.int64)
        for i in range(n * n):
            qx, qy = int(order[i]) % n, int(order[i]) // n
            x_lo = min(max(qx - w // 2, 0), n - w)
            y_lo = min(max(qy - w // 2, 0), n - w)
            for j in range(n * n):
                kx, ky = int(order[j]) % n, int(order[j]) // n
                if x_lo <= kx < x_lo + w and y_lo <= ky < y_lo + w:
                    cnt[i // block, j // block] += 1
        want = np.where(cnt == 0, 0, np.where(cnt == block * block, 2, 1))
        got = ho.block_classes(n, w, order, block)
        assert np.array_equal(got, want)
        assert (got == 1).any() and (got == 0).any()


@pytest.mark.parametrize("n", [2, 4, 8, 16, 64])
def test_curve_is_a_continuous_permutation(n):
    order = ho.hilbert_order(n)
    assert sorted(order.tolist()) == list(range(n * n))
    ys, xs = order // n, order % n
    steps = np.abs(np.diff(xs)) + np.abs(np.diff(ys))
    assert (steps == 1).all()                       # every step moves to a 4-neighbour
    assert (xs[0], ys[0]) == (0, 0) and (xs[-1], ys[-1]) == (n - 1, 0)


def test_smallest_curve_and_quadrants():
    assert [ho.hilbert_d2xy(2, d) for d in range(4)] == [(0, 0), (0, 1), (1, 1), (1, 0)]
    n = 16
    order = ho.hilbert_order(n)
    q = n * n // 4
    for k in range(4):                               # each quarter fills one quadrant
        ys, xs = order[k * q:(k + 1) * q] // n, order[k * q:(k + 1) * q] % n
        assert xs.max() - xs.min() == n // 2 - 1 and ys.max() - ys.min() == n // 2 - 1


def test_hilbert_blocks_are_rectangles():
    n = 64
    order = ho.hilbert_order(n)
    for b in range(n * n // 128):
        ys, xs = order[b * 128:(b + 1) * 128] // n, order[b * 128:(b + 1) * 128] % n
        w, h = xs.max() - xs.min() + 1, ys.max() - ys.min() + 1
        assert w * h == 128 and {w, h} == {8, 16}


def test_block_classes_special_cases():
    n = 32
    for order in (ho.raster_order(n), ho.hilbert_order(n)):
        assert (ho.block_classes(n, n, order) == 2).all()       # window covers the grid
        c1 = ho.block_classes(n, 1, order)                      # each query sees itself
        assert (np.diag(c1) == 1).all() and (c1 - np.diag(np.diag(c1)) == 0).all()


def test_rectangle_count_equals_brute_force():
    n = 64
    for w in (1, 9, 40):
        for order in (ho.raster_order(n), ho.hilbert_order(n)):
            assert (ho.block_classes_rect(n, w, order) == ho.block_classes(n, w, order)).all()


def test_hilbert_order_has_fewer_nonempty_and_partial_blocks():
    # the blog page's claim, for images wider than a 128-token block
    # (a raster block is then a fragment of one row)
    n = 256
    for w in (9, 21):
        r = ho.block_classes_rect(n, w, ho.raster_order(n))
        h = ho.block_classes_rect(n, w, ho.hilbert_order(n))
        assert (h > 0).sum() * 2 < (r > 0).sum()
        assert (h == 1).sum() * 2 < (r == 1).sum()


def test_attention_is_equivariant_under_the_order():
    # slide attention in Hilbert order = the raster result permuted
    n, w, d = 16, 5, 8
    rng = np.random.default_rng(0)
    q, k, v = (rng.standard_normal((n * n, d)) for _ in range(3))
    raster, _ = swa3d_oracle.swa3d_forward_rows(q, k, v, 1, n, n, (1, w, w), 0, False)
    order = ho.hilbert_order(n)
    mask = ho.slide_mask(n, w, order)
    qo, ko, vo = q[order], k[order], v[order]
    s = qo @ ko.T / np.sqrt(d)
    s = np.where(mask, s, -np.inf)
    p = np.exp(s - s.max(1, keepdims=True))
    o = (p @ vo) / p.sum(1, keepdims=True)
    np.testing.assert_allclose(o, raster[order], atol=1e-12)
