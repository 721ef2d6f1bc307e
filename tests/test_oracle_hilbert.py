"""Pins of the oracle's Hilbert key and sort (C1, C2) against properties the
definition fixes, independent of the oracle's own code.

Source: "Ab Initio Accuracy Beyond the Cutoff" (Tessera), abstract -- atoms
are sorted along a space-filling curve; the curve is the 3-D Hilbert curve
computed with Skilling's transform ("Programming the Hilbert curve", 2004).
"""
import itertools
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _grid(bits):
    return np.array(list(itertools.product(range(1 << bits), repeat=3)), dtype=np.uint32)


def test_one_bit_order_matches_hand_derived_table():
    want = np.loadtxt(os.path.join(GOLDEN, "hilbert_order_b1.txt"), dtype=np.int64)
    q = _grid(1)
    keys = oracle.hilbert_index_grid(q, 1)
    got = np.empty((8, 3), dtype=np.int64)
    got[keys] = q
    assert np.array_equal(got, want)
    # the table itself is a Gray-code walk: one axis flips per step
    assert np.all(np.abs(np.diff(want, axis=0)).sum(axis=1) == 1)


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 5, 6])
def test_bijection_unit_steps_and_origin(bits):
    q = _grid(bits)
    keys = oracle.hilbert_index_grid(q, bits)
    m = 1 << (3 * bits)
    assert keys.max() < m
    assert len(np.unique(keys)) == m                      # bijection
    inv = np.empty((m, 3), dtype=np.int64)
    inv[keys] = q
    assert np.all(inv[0] == 0)                            # starts at the origin
    steps = np.abs(np.diff(inv, axis=0)).sum(axis=1)
    assert np.all(steps == 1)                             # continuous: unit L1 steps


@pytest.mark.parametrize("bits", [2, 3, 4, 5])
def test_nested_subcubes_are_contiguous(bits):
    """Every aligned sub-cube of side 2^k occupies one contiguous key range
    of length 8^k -- the defining recursion of the Hilbert curve."""
    q = _grid(bits)
    keys = oracle.hilbert_index_grid(q, bits).astype(np.int64)
    for k in range(1, bits):
        cube = (q >> k).astype(np.int64)
        cid = (cube[:, 0] << 20) | (cube[:, 1] << 10) | cube[:, 2]
        blk = keys >> (3 * k)
        # one key block per sub-cube and one sub-cube per key block
        pairs = np.unique(np.stack([cid, blk], axis=1), axis=0)
        assert len(pairs) == len(np.unique(cid)) == len(np.unique(blk))


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 7])
def test_prefix_consistency(bits):
    """Dropping the last level of the key gives the coarser curve."""
    q = _grid(bits) if bits <= 6 else np.random.default_rng(1).integers(0, 1 << bits, (200000, 3)).astype(np.uint32)
    a = oracle.hilbert_index_grid(q, bits) >> 3
    b = oracle.hilbert_index_grid(q >> 1, bits - 1)
    assert np.array_equal(a, b)


def test_ten_bit_random_walk_steps():
    """At the working width (10 bits): consecutive keys are grid neighbors.
    Sample keys k, find both grid points by coarse-to-fine descent using the
    nesting property checked above, and compare."""
    rng = np.random.default_rng(7)
    bits = 10
    # points of a random 7-bit sub-block are enough to find consecutive keys:
    # take random points, and their 26 grid neighbors; any neighbor whose key is
    # key+1 must exist for every point except the last one on the curve.
    pts = rng.integers(1, (1 << bits) - 1, size=(20000, 3)).astype(np.int64)
    offs = np.array([o for o in itertools.product((-1, 0, 1), repeat=3) if sum(map(abs, o)) == 1], dtype=np.int64)
    k0 = oracle.hilbert_index_grid(pts.astype(np.uint32), bits).astype(np.int64)
    nb = (pts[:, None, :] + offs[None, :, :]).reshape(-1, 3)
    kn = oracle.hilbert_index_grid(nb.astype(np.uint32), bits).astype(np.int64).reshape(len(pts), 6)
    # the successor and the predecessor of every interior key is a unit step away
    assert np.all((kn == (k0 + 1)[:, None]).any(axis=1))
    assert np.all((kn == (k0 - 1)[:, None]).any(axis=1) | (k0 == 0))


def test_quantize_fp32_decision():
    L = np.float32(467.84283)
    assert oracle.quantize(0.0, L, 10) == 0
    assert oracle.quantize(np.nextafter(L, np.float32(0)), L, 10) == 1023
    assert oracle.quantize(L / 2, L, 10) == 512
    assert oracle.quantize(-1.0, L, 10) == 0                 # clamped
    assert oracle.quantize(float("nan"), L, 10) == 0
    assert oracle.quantize(2 * L, L, 10) == 1023             # clamped
    # the decision is the fp32 product, not the exact quotient
    s = np.float32(1024.0) / L
    x = np.float32(200.0)
    assert oracle.quantize(x, L, 10) == int(np.floor(np.float32(x * s)))


def test_sort_is_stable_total_order():
    rng = np.random.default_rng(3)
    L = (20.0, 20.0, 20.0)
    # coarse grid (bits=2) forces many equal keys
    pos = rng.uniform(0, 20, size=(5000, 3)).astype(np.float32)
    perm, keys = oracle.hilbert_sort(pos, L, bits=2)
    assert np.array_equal(np.sort(perm), np.arange(5000))
    k_all = oracle.hilbert_keys(pos, L, bits=2)
    assert np.array_equal(keys, k_all[perm])
    assert np.all(np.diff(keys.astype(np.int64)) >= 0)
    same = np.diff(keys.astype(np.int64)) == 0
    assert np.all(np.diff(perm)[same] > 0)                  # ties by ascending index
    # and agrees with numpy's stable sort of the same keys
    assert np.array_equal(perm, np.argsort(k_all, kind="stable"))


# ---------------------------------------------------------------- Morton (comparison curve)


def test_morton_hand_values():
    # the interleave read MSB-first, x's bit first: (1,0,0) at 1 bit is 0b100
    assert oracle.morton_index(1, 0, 0, 1) == 4
    assert oracle.morton_index(0, 1, 1, 1) == 3
    assert oracle.morton_index(3, 0, 0, 2) == 0b100100
    assert oracle.morton_index(0, 0, 3, 2) == 0b001001
    assert oracle.morton_index(1023, 1023, 1023, 10) == (1 << 30) - 1


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 5])
def test_morton_bijection_nesting_and_jumps(bits):
    q = _grid(bits)
    keys = oracle.morton_index_grid(q, bits).astype(np.int64)
    assert len(np.unique(keys)) == len(keys) == 1 << (3 * bits)
    for k in range(1, bits):
        cube = (q >> k).astype(np.int64)
        cid = (cube[:, 0] << 20) | (cube[:, 1] << 10) | cube[:, 2]
        pairs = np.unique(np.stack([cid, keys >> (3 * k)], axis=1), axis=0)
        assert len(pairs) == len(np.unique(cid))
    # unlike the Hilbert curve, the Z-order curve jumps: consecutive keys can
    # be far apart (from the top of one octant to the next)
    inv = np.empty((1 << (3 * bits), 3), dtype=np.int64)
    inv[keys] = q
    steps = np.abs(np.diff(inv, axis=0)).sum(axis=1)
    if bits >= 2:
        assert steps.max() > 1


def test_morton_sort_is_stable():
    rng = np.random.default_rng(5)
    pos = rng.uniform(0, 20, (4000, 3)).astype(np.float32)
    perm, keys = oracle.morton_sort(pos, (20, 20, 20), bits=2)
    q = np.stack([np.array([oracle.quantize(x, 20.0, 2) for x in pos[:, d]]) for d in range(3)], 1)
    k_all = oracle.morton_index_grid(q, 2)
    assert np.array_equal(perm, np.argsort(k_all, kind="stable"))
    assert np.array_equal(keys, k_all[perm])
