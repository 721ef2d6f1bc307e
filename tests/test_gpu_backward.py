"""GPU parity of the aggregation's backward (tess_edge_aggregate_backward)
against the oracle's plain chain rule, on lists built by the library.

Tolerances: the feature gradient is the forward aggregation of g over the
full symmetric list, so it gets the aggregate's condition-aware 1e-5; the
position gradient sums f_c'(r) (g_i.h_j + g_j.h_i) over edges, each a
length-F dot product in fp32, so it is compared per component against
1e-5 times its own magnitude scale sum_j |f_c'| (|g_i||h_j| + |g_j||h_i|)."""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import agg_error, torch_cuda

pytestmark = pytest.mark.gpu


def _dev(a):
    torch = torch_cuda()
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _case(s, F, seed, cap=None):
    import space_filling_curve_b200 as tess
    cap = s.cap if cap is None else cap
    perm, _ = oracle.hilbert_sort(s.pos, s.box, 10)
    p4 = s.pos4()[perm]
    rng = np.random.default_rng(seed)
    feat = rng.standard_normal((s.n, F)).astype(np.float32)
    g = rng.standard_normal((s.n, F)).astype(np.float32)
    nbr_d, cnt_d, ov = tess.build_neighbors(_dev(p4), s.box, s.rc, s.skin, cap)
    assert int(ov.item()) == 0
    gf, gp = tess.edge_aggregate_backward(_dev(p4), s.box, s.rc, nbr_d, cnt_d, _dev(feat), _dev(g))
    nbr, cnt = nbr_d.cpu().numpy(), cnt_d.cpu().numpy()
    ogf, ogp = oracle.edge_backward(p4, s.box, s.rc, nbr, cnt, feat, g)
    # feature gradient: the forward of g, with its conditioning
    ref = oracle.edge_aggregate(p4, s.box, s.rc, nbr, cnt, g)
    assert np.allclose(ref["out"], ogf, rtol=1e-12, atol=1e-12)
    err, _ = agg_error(gf.cpu().numpy(), ref)
    assert err <= 1e-5
    # position gradient: per-row magnitude scale of the sum
    e = oracle.edge_aggregate(p4, s.box, s.rc, nbr, cnt, np.ones((s.n, 1), np.float32), edges=True)
    r = e["edge_vec"][..., 3]
    i_idx = np.repeat(np.arange(s.n), cap).reshape(s.n, cap)
    live = (np.arange(cap)[None, :] < np.minimum(cnt, cap)[:, None]) & (r < s.rc) & (nbr >= 0)
    ii, jj = i_idx[live], nbr[live]
    dfc = np.abs(-0.5 * np.pi / s.rc * np.sin(np.pi * r[live] / s.rc))
    gn = np.linalg.norm(g.astype(np.float64), axis=1)
    hn = np.linalg.norm(feat.astype(np.float64), axis=1)
    scale = np.zeros(s.n)
    np.add.at(scale, ii, dfc * (gn[ii] * hn[jj] + gn[jj] * hn[ii]))
    diff = np.abs(gp.cpu().numpy().astype(np.float64) - ogp)
    assert np.all(diff <= 1e-5 * scale[:, None] + 1e-12)
    # translation invariance survives fp32 to well within the same scale
    assert np.abs(gp.cpu().numpy().astype(np.float64).sum(0)).max() <= 1e-5 * scale.sum()


@pytest.mark.parametrize("F", [4, 8, 32, 64, 128])
def test_backward_uniform(F):
    _case(synth.system(1), F, F)


def test_backward_salt():
    _case(synth.system(2), 64, 7)


def test_backward_large_cap():
    """cap 512: the staging buffers of a block exceed the default 48 KB of
    dynamic shared memory."""
    _case(synth.system(1), 32, 9, cap=512)


def test_backward_rejects_unsupported_widths():
    import space_filling_curve_b200 as tess
    s = synth.system(1)
    p = _dev(s.pos4())
    nbr, cnt, _ = tess.build_neighbors(p, s.box, s.rc, s.skin, s.cap)
    f = _dev(np.zeros((s.n, 12), np.float32))
    with pytest.raises(tess.TessError):
        tess.edge_aggregate_backward(p, s.box, s.rc, nbr, cnt, f, f)
