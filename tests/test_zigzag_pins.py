"""Pins for the zigzag scan orders (codes 4..11) of the oracle, and the GLA over them.

ZigMa notes, "Zigzag 扫描方案": the scan turns back at the end of every line (a
snake path), so tokens adjacent in the sequence are adjacent in the grid; eight
schemes S_0..S_7 differ in orientation (rows or columns), start and direction.
The reading (oracle/dig_oracle.c, zigzag_order): S_j walks rows for j < 4 and
columns for j >= 4, lines last-to-first when bit 1 of j is set, the first line from
its end when bit 0 is set.  Pinned here by closed-form index formulas, the
adjacency property that defines a zigzag, the start corners, the eight schemes
being the images of S_0 under the eight symmetries of a square grid, and the O(T^2)
brute force of the GLA along each order.
"""
import numpy as np
import pytest

import oracle

from test_oracle_pins import bruteforce, rand_inputs, zigzag_closed_form

GRIDS = [(3, 4), (4, 3), (5, 5), (1, 6), (6, 1), (1, 1), (2, 7), (16, 16), (7, 13)]


@pytest.mark.parametrize("Hg,Wg", GRIDS)
@pytest.mark.parametrize("j", range(8))
def test_zigzag_closed_form_bijection_adjacency(Hg, Wg, j):
    order = oracle.scan_order(4 + j, Hg, Wg)
    assert np.array_equal(order, zigzag_closed_form(j, Hg, Wg))
    assert np.array_equal(np.sort(order), np.arange(Hg * Wg))
    y, x = order // Wg, order % Wg
    steps = np.abs(np.diff(y)) + np.abs(np.diff(x))
    assert np.all(steps == 1), "consecutive tokens must be grid neighbours"


@pytest.mark.parametrize("Hg,Wg", [(3, 4), (5, 2), (4, 4)])
def test_zigzag_start_corners(Hg, Wg):
    corners = {0: (0, 0), 1: (0, Wg - 1), 2: (Hg - 1, 0), 3: (Hg - 1, Wg - 1),
               4: (0, 0), 5: (Hg - 1, 0), 6: (0, Wg - 1), 7: (Hg - 1, Wg - 1)}
    for j, (y, x) in corners.items():
        order = oracle.scan_order(4 + j, Hg, Wg)
        assert order[0] == y * Wg + x
        # rows schemes move along the row first, column schemes along the column
        dy, dx = divmod(int(order[1]), Wg)[0] - y, int(order[1]) % Wg - x
        assert (dy == 0) == (j < 4)


@pytest.mark.parametrize("n", [2, 3, 4, 6])
def test_zigzag_schemes_are_the_square_symmetries_of_s0(n):
    """On an n x n grid the eight schemes are exactly S_0 mapped by the eight
    symmetries of the square (four rotations, four reflections)."""
    s0 = oracle.scan_order(4, n, n)
    ys, xs = s0 // n, s0 % n
    maps = [lambda y, x: (y, x), lambda y, x: (y, n - 1 - x), lambda y, x: (n - 1 - y, x),
            lambda y, x: (n - 1 - y, n - 1 - x), lambda y, x: (x, y), lambda y, x: (x, n - 1 - y),
            lambda y, x: (n - 1 - x, y), lambda y, x: (n - 1 - x, n - 1 - y)]
    images = set()
    for m in maps:
        yy, xx = m(ys, xs)
        images.add(tuple((yy * n + xx).tolist()))
    schemes = {tuple(oracle.scan_order(4 + j, n, n).tolist()) for j in range(8)}
    assert len(schemes) == 8
    assert schemes == images


@pytest.mark.parametrize("Hg,Wg", [(3, 4), (2, 5), (4, 4)])
@pytest.mark.parametrize("j", range(8))
def test_gla_along_zigzag_matches_bruteforce(Hg, Wg, j):
    rng = np.random.default_rng(100 + j)
    q, k, v, la = rand_inputs(rng, 1, 2, Hg, Wg, 3, 4)
    got = oracle.gla_fwd(q, k, v, la, Hg, Wg, 4 + j, nthreads=1)
    np.testing.assert_allclose(got, bruteforce(q, k, v, la, Hg, Wg, 4 + j), rtol=1e-12, atol=1e-12)


def test_reorient_along_zigzag_is_the_order_gather():
    x = np.arange(2 * 12 * 3, dtype=np.int32).reshape(2, 12, 3)
    for j in range(8):
        order = zigzag_closed_form(j, 3, 4)
        y = oracle.reorient(x, 4 + j, 0, 3, 4)
        assert np.array_equal(y, x[:, order])
        assert np.array_equal(oracle.reorient(y, 4 + j, 1, 3, 4), x)
