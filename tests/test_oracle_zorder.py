"""Pins for the oracle's quadtree (Z) token order, on CPU: a recursive quadrant
construction written independently of the oracle's bit interleave, bijection, and the
round trip."""
import os

import numpy as np
import pytest

from oracle.llsa_oracle import from_z_order, to_z_order, zorder_index


def quadrants(side):
    """Row-major grid of indices filled quadrant by quadrant: top-left, top-right,
    bottom-left, bottom-right, each filled the same way, recursively."""
    if side == 1:
        return np.zeros((1, 1), dtype=np.int64)
    h = side // 2
    sub = quadrants(h)
    grid = np.empty((side, side), dtype=np.int64)
    grid[:h, :h] = sub
    grid[:h, h:] = sub + h * h
    grid[h:, :h] = sub + 2 * h * h
    grid[h:, h:] = sub + 3 * h * h
    return grid


@pytest.mark.parametrize("side", [1, 2, 4, 8, 16, 64])
def test_zorder_matches_recursive_quadrants(side):
    assert np.array_equal(zorder_index(side), quadrants(side).ravel())


@pytest.mark.parametrize("side", [2, 16, 256])
def test_zorder_is_a_bijection(side):
    z = zorder_index(side)
    assert np.array_equal(np.sort(z), np.arange(side * side))


def test_first_quadrant_order():
    # the four cells of a 2 x 2 grid: (0,0), (0,1), (1,0), (1,1) -> 0, 1, 2, 3
    assert zorder_index(2).tolist() == [0, 1, 2, 3]
    # on 4 x 4 the top-right 2 x 2 quadrant holds 4..7
    assert sorted(zorder_index(4).reshape(4, 4)[:2, 2:].ravel().tolist()) == [4, 5, 6, 7]


def test_round_trip_and_neighbourhoods():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((2, 3, 1024, 5))
    z = to_z_order(x)
    assert np.array_equal(from_z_order(z), x)
    # each run of 16 Z-ordered tokens is a 4 x 4 square of the grid
    side = 32
    pos = np.argsort(zorder_index(side))  # grid position of each Z index
    r, c = np.divmod(pos.reshape(-1, 16), side)
    assert np.all(r.max(1) - r.min(1) == 3) and np.all(c.max(1) - c.min(1) == 3)
    with pytest.raises(ValueError):
        to_z_order(np.zeros((1, 1, 8, 2)))


def _golden_zorder():
    """Sections of tests/golden/zorder_grid_4x4.txt (values from the README's token
    reordering example; see the file's header)."""
    path = os.path.join(os.path.dirname(__file__), "golden", "zorder_grid_4x4.txt")
    sections, name = {}, None
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        if line[0].isalpha():
            name = line
            sections[name] = []
        else:
            sections[name].append([int(t) for t in line.split()])
    return {k: np.array(v) for k, v in sections.items()}


def test_zorder_matches_the_readme_example():
    g = _golden_zorder()
    assert np.array_equal(zorder_index(2).reshape(2, 2), g["grid2"])
    assert np.array_equal(zorder_index(4).reshape(4, 4), g["grid4"])
    tokens = np.arange(16, dtype=np.float64).reshape(1, 1, 16, 1)
    assert np.array_equal(to_z_order(tokens)[0, 0, :, 0].astype(int), g["order4"][0])
