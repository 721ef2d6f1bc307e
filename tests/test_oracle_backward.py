"""Pins of the oracle's backward (VJP) of the aggregation against finite
differences of the forward oracle and against identities of the full list.

The forces come from a backward pass through every layer, which repeats the
neighbor exchange ("Ab Initio Accuracy Beyond the Cutoff" (Tessera),
abstract): forces are -dE/dr; this is the one-hop aggregation's share of that
chain rule.
"""
import numpy as np
import pytest

import oracle
import synth


def _setup(seed=0, n=400, L=16.0, F=5):
    rng = np.random.default_rng(seed)
    pos = np.zeros((n, 4), np.float32)
    pos[:, :3] = rng.uniform(0, L, (n, 3))
    box = (L, L, L)
    rc, skin = 4.0, 0.5
    nbr, cnt, ov = oracle.neighbors_brute(pos, box, rc, skin, 256)
    assert ov == 0
    feat = rng.standard_normal((n, F)).astype(np.float32)
    g = rng.standard_normal((n, F)).astype(np.float32)
    return pos, box, rc, nbr, cnt, feat, g


def _loss(pos, box, rc, nbr, cnt, feat, g):
    out = oracle.edge_aggregate(pos, box, rc, nbr, cnt, feat)["out"]
    return float((out * g.astype(np.float64)).sum())


def test_cutoff_derivative_closed_forms():
    rc = 5.75
    assert oracle.cutoff_deriv(0.0, rc) == 0.0
    assert oracle.cutoff_deriv(rc / 2, rc) == pytest.approx(-np.pi / (2 * rc), rel=1e-15)
    assert oracle.cutoff_deriv(rc, rc) == 0.0
    h = 1e-6
    for r in (0.7, 2.0, 4.9):
        fd = (oracle.cutoff(r + h, rc) - oracle.cutoff(r - h, rc)) / (2 * h)
        assert oracle.cutoff_deriv(r, rc) == pytest.approx(fd, rel=1e-6)


def test_feature_gradient_is_linear_and_matches_the_forward_of_g():
    pos, box, rc, nbr, cnt, feat, g = _setup()
    gf, _ = oracle.edge_backward(pos, box, rc, nbr, cnt, feat, g)
    # L is linear in h: dL/dh_j[f] is exact from one unit perturbation
    for j, f in ((3, 0), (100, 4), (399, 2)):
        e = np.zeros_like(feat)
        e[j, f] = 1.0
        d = _loss(pos, box, rc, nbr, cnt, feat + e, g) - _loss(pos, box, rc, nbr, cnt, feat, g)
        assert gf[j, f] == pytest.approx(d, rel=1e-9, abs=1e-9)
    # a full symmetric list makes the feature gradient the forward of g
    fwd = oracle.edge_aggregate(pos, box, rc, nbr, cnt, g)["out"]
    assert np.allclose(gf, fwd, rtol=1e-12, atol=1e-12)


def test_position_gradient_matches_central_differences():
    pos, box, rc, nbr, cnt, feat, g = _setup(seed=1)
    _, gp = oracle.edge_backward(pos, box, rc, nbr, cnt, feat, g)
    # central differences on fp32 coordinates (step a few hundred ulps at L = 16)
    eps = np.float32(1e-3)
    for i, a in ((0, 0), (17, 1), (250, 2)):
        p1 = pos.copy(); p1[i, a] += eps
        p0 = pos.copy(); p0[i, a] -= eps
        step = float(p1[i, a]) - float(p0[i, a])
        fd = (_loss(p1, box, rc, nbr, cnt, feat, g) - _loss(p0, box, rc, nbr, cnt, feat, g)) / step
        assert gp[i, a] == pytest.approx(fd, rel=2e-4, abs=2e-5)


def test_position_gradient_sums_to_zero():
    # translating every atom changes nothing: the gradients sum to zero
    pos, box, rc, nbr, cnt, feat, g = _setup(seed=2)
    _, gp = oracle.edge_backward(pos, box, rc, nbr, cnt, feat, g)
    assert np.allclose(gp.sum(axis=0), 0.0, atol=1e-9 * np.abs(gp).sum())
