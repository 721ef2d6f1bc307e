"""Pins of the oracle's closest-listed-pair monitor (oracle.min_pair).

Tessera's long runs were checked for atoms that come anomalously close
("Ab Initio Accuracy Beyond the Cutoff" (Tessera), abstract); the monitor
reports the closest pair the neighbor list holds.  Pinned by an
independent all-pairs brute force (numpy, minimum image by rounding), a
hand case across a periodic face, ties, an empty list and overflowed rows.
"""
import numpy as np

import oracle
import synth


def _brute(pos, box):
    p = pos.astype(np.float64)
    L = np.asarray(box, dtype=np.float64)
    best = (np.inf, -1, -1)
    for i in range(len(p) - 1):
        d = p[i + 1:] - p[i]
        d -= L * np.round(d / L)
        r2 = (d[:, 0] * d[:, 0] + d[:, 1] * d[:, 1]) + d[:, 2] * d[:, 2]
        k = int(np.argmin(r2))
        if r2[k] < best[0]:
            best = (float(r2[k]), i, i + 1 + k)
    return best


def test_matches_all_pairs_brute_force():
    s = synth.system(1)
    nbr, cnt, ov = oracle.neighbors_cells(s.pos, s.box, s.rc, s.skin, s.cap)
    assert ov == 0
    r2, i, j = oracle.min_pair(s.pos, s.box, nbr, cnt)
    b = _brute(s.pos, s.box)
    assert r2 == b[0] and (i, j) == (b[1], b[2])
    assert r2 >= 0.9 ** 2 * (1 - 1e-6)          # the generator's minimum separation


def test_hand_case_across_a_face():
    box = (10.0, 10.0, 10.0)
    pos = np.array([[5.0, 5.0, 5.0], [9.9, 5.0, 5.0], [0.2, 5.0, 5.0], [5.0, 7.5, 5.0]], np.float32)
    nbr, cnt, _ = oracle.neighbors_brute(pos, box, 3.0, 0.0, 8)
    r2, i, j = oracle.min_pair(pos, box, nbr, cnt)
    dx = (np.float64(np.float32(0.2)) - np.float64(np.float32(9.9))) + 10.0
    assert (i, j) == (1, 2)
    assert r2 == dx * dx
    assert abs(np.sqrt(r2) - 0.3) < 1e-6


def test_ties_go_to_the_smallest_pair():
    box = (20.0, 20.0, 20.0)
    # a square of side 2: four sides tie, the diagonals are longer
    pos = np.array([[5, 5, 5], [7, 5, 5], [7, 7, 5], [5, 7, 5]], np.float32)
    nbr, cnt, _ = oracle.neighbors_brute(pos, box, 4.0, 0.0, 8)
    assert oracle.min_pair(pos, box, nbr, cnt) == (4.0, 0, 1)
    # reversed atom order: the tie still goes to the smallest (i, j)
    nbr, cnt, _ = oracle.neighbors_brute(pos[::-1].copy(), box, 4.0, 0.0, 8)
    assert oracle.min_pair(pos[::-1].copy(), box, nbr, cnt) == (4.0, 0, 1)


def test_nothing_listed():
    pos = np.array([[1, 1, 1], [9, 9, 9]], np.float32)
    nbr = np.full((2, 4), -1, np.int32)
    cnt = np.zeros(2, np.int32)
    r2, i, j = oracle.min_pair(pos, (20.0, 20.0, 20.0), nbr, cnt)
    assert r2 == np.inf and (i, j) == (-1, -1)


def test_only_stored_entries_count():
    box = (20.0, 20.0, 20.0)
    pos = np.array([[5, 5, 5], [6, 5, 5], [5.5, 5, 5]], np.float32)
    # row 0 claims two neighbors but stores only atom 1; row 1 stores only 0
    nbr = np.array([[1], [0], [-1]], np.int32)
    cnt = np.array([2, 1, 0], np.int32)
    assert oracle.min_pair(pos, box, nbr, cnt) == (1.0, 0, 1)
