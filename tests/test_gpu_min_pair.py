"""GPU parity of the closest-listed-pair monitor (tess_min_pair_distance)
against the oracle on the same list: the squared distance bit for bit
(both fp64 from the fp32 coordinates, one rounding per operation) and the
same pair (ties to the smallest (i, j))."""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import torch_cuda

pytestmark = pytest.mark.gpu


def _dev(a):
    torch = torch_cuda()
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _check(pos4, box, nbr, cnt):
    import space_filling_curve_b200 as tess
    r2, pair = tess.min_pair_distance(_dev(pos4), box, _dev(nbr), _dev(cnt))
    want = oracle.min_pair(pos4, box, nbr, cnt)
    got = (float(r2.item()), *[int(x) for x in pair.cpu().numpy()])
    assert got == want, (got, want)
    return got


@pytest.mark.parametrize("cfg", [1, 2, 3])
def test_min_pair_on_built_lists(cfg):
    import space_filling_curve_b200 as tess
    s = synth.system(cfg)
    p4 = s.pos4()
    nbr, cnt, ov = tess.build_neighbors(_dev(p4), s.box, s.rc, s.skin, s.cap)
    assert int(ov.item()) == 0
    _check(p4, s.box, nbr.cpu().numpy(), cnt.cpu().numpy())


def test_planted_close_pair_and_ties():
    s = synth.system(1)
    p4 = s.pos4().copy()
    # atom 7 placed 0.05 A from atom 3 (across x if near a face), atom 11 at
    # the same distance from atom 5: two pairs tie, the smaller one wins
    L = np.array(s.box, np.float64)
    for a, b in ((3, 7), (5, 11)):
        x = p4[a, :3].astype(np.float64) + np.array([0.05, 0.0, 0.0])
        p4[b, :3] = synth.wrap_cast(x[None, :], s.box)[0]
    nbr, cnt, _ = oracle.neighbors_cells(p4, s.box, s.rc, s.skin, 256)
    r2, i, j = _check(p4, s.box, nbr, cnt)
    assert (i, j) in ((3, 7), (5, 11)) and r2 < 0.06 ** 2


def test_min_pair_empty_and_overflowed():
    s = synth.system(1)
    p4 = s.pos4()
    nbr = np.full((s.n, 4), -1, np.int32)
    cnt = np.zeros(s.n, np.int32)
    assert _check(p4, s.box, nbr, cnt) == (float("inf"), -1, -1)
    # rows cut at 3 entries: only the stored entries count
    full, fcnt, _ = oracle.neighbors_cells(p4, s.box, s.rc, s.skin, s.cap)
    _check(p4, s.box, np.ascontiguousarray(full[:, :3]), fcnt)


def test_min_pair_full_size():
    import space_filling_curve_b200 as tess
    s = synth.system(4)
    perm, keys, ps, _ = tess.hilbert_sort(_dev(s.pos), s.box)
    nbr, cnt, ov = tess.build_neighbors(ps, s.box, s.rc, s.skin, s.cap)
    assert int(ov.item()) == 0
    _check(ps.cpu().numpy(), s.box, nbr.cpu().numpy(), cnt.cpu().numpy())
