"""Pins of the oracle's Verlet list (C3), skin check (C4) and edge
aggregation (C5) against hand examples, closed forms, invariants and the
agreement of two independent methods.

Sources: "Ab Initio Accuracy Beyond the Cutoff" (Tessera), abstract (fixed
shapes between rebuilds, conservative neighbor skin); review of arXiv
2505.06711, "load-bearing attack" paragraph (one-hop aggregation within the
original cutoff).
"""
import numpy as np
import pytest

import oracle
import synth


def _pos(*xyz):
    return np.array(xyz, dtype=np.float32).reshape(-1, 3)


# --------------------------------------------------------------------- C3


def test_two_atoms_across_the_boundary():
    # L = 20, atoms at x = 0.5 and 19.0: the minimum image is 1.5 apart
    pos = _pos(0.5, 5, 5, 19.0, 5, 5)
    for fn in (oracle.neighbors_brute, oracle.neighbors_cells):
        nbr, cnt, ov = fn(pos, (20, 20, 20), 6.0, 0.5, 4)
        assert cnt.tolist() == [1, 1] and ov == 0
        assert nbr.tolist() == [[1, -1, -1, -1], [0, -1, -1, -1]]


@pytest.mark.parametrize("d,inside", [(6.4, True), (6.6, False), (6.499, True), (6.501, False)])
def test_radius_is_rc_plus_skin(d, inside):
    pos = _pos(1.0, 10, 10, 1.0 + d, 10, 10)
    nbr, cnt, _ = oracle.neighbors_brute(pos, (30, 30, 30), 6.0, 0.5, 2)
    assert cnt.tolist() == ([1, 1] if inside else [0, 0])


def test_square_across_a_periodic_corner():
    # four atoms at the corners of a 2 A square that straddles the corner of
    # the box: every pair is within rs, each atom has the other three
    L = 25.0
    pos = _pos(24.0, 24.0, 3.0, 1.0, 24.0, 3.0, 24.0, 1.0, 3.0, 1.0, 1.0, 3.0)
    for fn in (oracle.neighbors_brute, oracle.neighbors_cells):
        nbr, cnt, _ = fn(pos, (L, L, L), 3.0, 0.5, 8)
        assert cnt.tolist() == [3, 3, 3, 3]
        for i in range(4):
            assert sorted(nbr[i, :3].tolist()) == [j for j in range(4) if j != i]


def test_distance_uses_all_three_axes_and_minimum_image():
    # displacement (3, 4, 0) -> 5 (in at rs 5.5), (3, 4, 3) -> 5.83 (out),
    # and the same displacements across each face
    L = 20.0
    for base in ((1.0, 1.0, 1.0), (18.5, 18.0, 19.5)):
        bx, by, bz = base
        pos = _pos(bx, by, bz, (bx + 3) % L, (by + 4) % L, bz, (bx - 3) % L, (by + 4) % L, (bz + 3) % L)
        nbr, cnt, _ = oracle.neighbors_brute(pos, (L, L, L), 5.0, 0.5, 4)
        r01 = 5.0
        r02 = np.sqrt(9 + 16 + 9)
        r12 = np.sqrt(36 + 0 + 9)
        want = [int(r01 < 5.5) + int(r02 < 5.5), int(r01 < 5.5) + int(r12 < 5.5), int(r02 < 5.5) + int(r12 < 5.5)]
        assert cnt.tolist() == want


def test_overflow_keeps_true_counts():
    sysm = synth.system(1)
    nbr, cnt, ov = oracle.neighbors_cells(sysm.pos, sysm.box, sysm.rc, sysm.skin, 16)
    full, fcnt, fov = oracle.neighbors_cells(sysm.pos, sysm.box, sysm.rc, sysm.skin, 400)
    assert ov == 1 and fov == 0
    assert np.array_equal(cnt, fcnt)
    # the stored entries are the cap smallest indices of each row
    assert np.array_equal(nbr, full[:, :16])


def _rows_as_sets(nbr, cnt):
    return [set(nbr[i, : min(c, nbr.shape[1])].tolist()) for i, c in enumerate(cnt)]


@pytest.mark.parametrize("which", ["uniform", "salt"])
def test_brute_equals_cells_and_symmetry(which):
    s = synth.system(1) if which == "uniform" else synth.custom("salt", 2000, rc=6.0, cap=192)
    a, ca, oa = oracle.neighbors_brute(s.pos, s.box, s.rc, s.skin, s.cap)
    b, cb, ob = oracle.neighbors_cells(s.pos, s.box, s.rc, s.skin, s.cap)
    assert oa == ob == 0
    assert np.array_equal(ca, cb) and np.array_equal(a, b)
    rows = _rows_as_sets(a, ca)
    for i, r in enumerate(rows):
        assert i not in r
        for j in r:
            assert i in rows[j]                           # j in N(i) <=> i in N(j)


def test_mean_count_matches_density():
    # uniform gas: mean count = rho * (4/3 pi rs^3 - excluded sphere of 0.9 A)
    s = synth.system(1)
    _, cnt, _ = oracle.neighbors_cells(s.pos, s.box, s.rc, s.skin, s.cap)
    rho = (s.n - 1) / np.prod(s.box)
    expect = 4.0 / 3.0 * np.pi * (s.rs ** 3 - 0.9 ** 3) * rho
    # mean of 3000 correlated Poisson-like counts: well within 2%
    assert abs(cnt.mean() - expect) / expect < 0.02
    # salt solution: molecular exclusion shifts the mean by a few percent
    s = synth.system(2)
    _, cnt, _ = oracle.neighbors_cells(s.pos, s.box, s.rc, s.skin, s.cap)
    expect = 4.0 / 3.0 * np.pi * s.rs ** 3 * s.n / np.prod(s.box)
    assert abs(cnt.mean() - expect) / expect < 0.06


def test_neighbors_of_matches_full_list():
    s = synth.system(1)
    nbr, cnt, _ = oracle.neighbors_brute(s.pos, s.box, s.rc, s.skin, s.cap)
    for i in (0, 17, 2999):
        row = oracle.neighbors_of(s.pos, s.box, s.rc, s.skin, i)
        assert row.tolist() == nbr[i, : cnt[i]].tolist()


def test_generated_inputs_have_no_pair_in_the_band():
    s = synth.system(1)
    nbr, cnt, _ = oracle.neighbors_brute(s.pos, s.box, s.rc, s.skin + 0.01, 400)
    i = np.repeat(np.arange(s.n), cnt)
    j = nbr[nbr >= 0]
    d = oracle.pair_distances(s.pos, s.box, i, j)
    assert np.all(np.abs(d - s.rs) >= 1e-4)
    assert d.min() >= 0.9


# --------------------------------------------------------------------- C4


@pytest.mark.parametrize("move,flag", [(0.26, 1), (0.24, 0), (0.250003, 1), (0.249997, 0), (0.25, 0)])
def test_skin_half_criterion(move, flag):
    ref = _pos(5, 5, 5, 10, 10, 10)
    pos = ref.copy()
    pos[1, 1] += np.float32(move)
    f, m = oracle.skin_check(pos, ref, (20, 20, 20), 0.5)
    assert f == flag
    d = float(np.float32(10 + np.float32(move)) - np.float32(10))
    assert m == pytest.approx(d * d, rel=0, abs=0)


def test_skin_across_the_boundary_uses_minimum_image():
    ref = _pos(19.9, 5, 5)
    pos = _pos(0.05, 5, 5)                       # moved +0.15 through the face
    f, m = oracle.skin_check(pos, ref, (20, 20, 20), 0.5)
    assert f == 0
    exact = (np.float64(np.float32(0.05)) - np.float64(np.float32(19.9)) + np.float64(np.float32(20.0))) ** 2
    assert m == exact


def test_skin_max_over_atoms():
    rng = np.random.default_rng(0)
    ref = rng.uniform(0, 30, (1000, 3)).astype(np.float32)
    pos = ref + rng.normal(0, 0.05, ref.shape).astype(np.float32)
    pos = np.mod(pos, np.float32(30)).astype(np.float32)
    f, m = oracle.skin_check(pos, ref, (30, 30, 30), 0.5)
    d = pos.astype(np.float64) - ref.astype(np.float64)
    d -= 30 * np.round(d / 30)
    assert m == pytest.approx((d * d).sum(1).max(), rel=1e-15)
    assert f == int(m > 0.0625)


# --------------------------------------------------------------------- C5


def test_cutoff_closed_forms():
    rc = 5.75
    assert oracle.cutoff(0.0, rc) == 1.0
    assert oracle.cutoff(rc / 2, rc) == pytest.approx(0.5, abs=1e-15)
    assert oracle.cutoff(rc, rc) == 0.0
    assert oracle.cutoff(rc + 1, rc) == 0.0
    # smooth at rc: slope -> 0 from below
    h = 1e-6
    assert abs(oracle.cutoff(rc - h, rc) - oracle.cutoff(rc - 2 * h, rc)) / h < 1e-5
    # decreasing on (0, rc)
    r = np.linspace(0, rc, 50)
    v = [oracle.cutoff(x, rc) for x in r]
    assert np.all(np.diff(v) <= 0)


def test_two_atom_aggregate_is_the_cutoff():
    pos = _pos(1.0, 1.0, 1.0, 3.0, 1.0, 1.0)
    nbr = np.array([[1, -1], [0, -1]], np.int32)
    cnt = np.array([1, 1], np.int32)
    feat = np.array([[2.0, -1.0], [1.0, 3.0]], np.float32)
    r = oracle.edge_aggregate(pos, (10, 10, 10), 5.0, nbr, cnt, feat, edges=True)
    fc = 0.5 * (np.cos(np.pi * 2.0 / 5.0) + 1)
    assert np.allclose(r["out"], [[fc * 1.0, fc * 3.0], [fc * 2.0, -fc]], rtol=0, atol=1e-15)
    assert np.allclose(r["edge_vec"][0, 0], [2, 0, 0, 2]) and np.allclose(r["edge_vec"][1, 0], [-2, 0, 0, 2])
    assert np.allclose(r["edge_unit"][0, 0], [1, 0, 0, 0]) and np.allclose(r["edge_unit"][1, 0], [-1, 0, 0, 0])
    assert r["edge_fc"][0, 1] == 0.0 and np.all(r["edge_vec"][0, 1] == 0)


def test_aggregate_identities():
    s = synth.system(1)
    nbr, cnt, _ = oracle.neighbors_cells(s.pos, s.box, s.rc, s.skin, s.cap)
    ones = np.ones((s.n, 1), np.float32)
    r1 = oracle.edge_aggregate(s.pos, s.box, s.rc, nbr, cnt, ones, edges=True)
    sum_fc = r1["edge_fc"].sum(axis=1)
    # constant features: out_i = c * sum_j f_c
    assert np.allclose(r1["out"][:, 0], sum_fc, rtol=1e-14, atol=0)
    h = s.features()
    r = oracle.edge_aggregate(s.pos, s.box, s.rc, nbr, cnt, h)
    # full symmetric list: sum_i out_i = sum_j h_j * (sum_i f_c(r_ij))
    lhs = r["out"].sum(axis=0)
    rhs = (h.astype(np.float64) * sum_fc[:, None]).sum(axis=0)
    assert np.allclose(lhs, rhs, rtol=1e-12, atol=1e-9)
    # edges beyond rc contribute nothing; f_c within [0, 1]
    ev, ef = r1["edge_vec"], r1["edge_fc"]
    assert np.all(ef[ev[..., 3] >= s.rc] == 0) and ef.max() <= 1 and ef.min() >= 0
    # the edge vector is the minimum image of r_j - r_i
    i = 5
    for slot in range(cnt[i]):
        j = nbr[i, slot]
        d = s.pos[j].astype(np.float64) - s.pos[i].astype(np.float64)
        d -= np.asarray(s.box) * np.round(d / np.asarray(s.box))
        assert np.allclose(ev[i, slot, :3], d, atol=1e-12)


def test_sampled_row_helpers_match_the_full_oracle():
    s = synth.system(1)
    nbr, cnt, _ = oracle.neighbors_brute(s.pos, s.box, s.rc, s.skin, s.cap)
    rows = np.array([0, 5, 17, 2999])
    r, rc = oracle.neighbors_rows(s.pos, s.box, s.rc, s.skin, rows, s.cap)
    assert np.array_equal(r, nbr[rows]) and np.array_equal(rc, cnt[rows])
    f = s.features()
    full = oracle.edge_aggregate(s.pos, s.box, s.rc, nbr, cnt, f)
    part = oracle.edge_aggregate_rows(s.pos, s.box, s.rc, nbr, cnt, f, rows)
    assert np.array_equal(full["out"][rows], part["out"])
    assert np.array_equal(full["out_abs"][rows], part["out_abs"])
