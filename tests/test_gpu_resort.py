"""GPU parity of the incremental re-sort (tess_hilbert_resort): whatever
earlier order it is given, its outputs must be exactly the oracle's full
Hilbert sort of the current positions (perm, keys and sorted positions, bit
for bit), and it must take its incremental path when the earlier order is a
recent sort of the same atoms."""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import torch_cuda

pytestmark = pytest.mark.gpu

FULL_SORT = 8


def _dev(a):
    torch = torch_cuda()
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _check(pos, box, perm_prev, keys_prev, bits=10, expect_fast=None):
    import space_filling_curve_b200 as tess
    perm, keys, ps, st = tess.hilbert_resort(_dev(pos), box, _dev(perm_prev), _dev(keys_prev), bits)
    want_perm, want_keys = oracle.hilbert_sort(pos, box, bits)
    assert np.array_equal(perm.cpu().numpy(), want_perm)
    assert np.array_equal(keys.cpu().numpy().view(np.uint32), want_keys.astype(np.uint32))
    want_ps = np.zeros((len(pos), 4), np.float32)
    want_ps[:, :3] = pos[want_perm]
    assert np.array_equal(ps.cpu().numpy(), want_ps)
    status = int(st.item())
    assert status & ~(FULL_SORT | 2) == 0
    if expect_fast is not None:
        assert bool(status & FULL_SORT) == (not expect_fast)
    return perm.cpu().numpy(), keys.cpu().numpy().view(np.uint32), status


def _wrap(x, box):
    return synth.wrap_cast(x, box)


def test_resort_along_a_trajectory():
    """Salt solution, 98,304 atoms: the earlier order is refreshed every 20
    steps (a rebuild interval); every step in between is re-sorted from it."""
    s = synth.system(2)
    perm_prev, keys_prev = oracle.hilbert_sort(s.pos, s.box, 10)
    fast = 0
    for t, p in s.trajectory(60, condition=False):
        perm, keys, st = _check(p, s.box, perm_prev.astype(np.int32), keys_prev.astype(np.uint32).view(np.int32))
        fast += not (st & FULL_SORT)
        if t % 20 == 0:
            perm_prev, keys_prev = perm, keys
    assert fast == 60


def test_resort_same_positions_is_fast_and_exact():
    s = synth.system(3)
    perm, keys = oracle.hilbert_sort(s.pos, s.box, 10)
    _check(s.pos, s.box, perm.astype(np.int32), keys.astype(np.uint32).view(np.int32), expect_fast=True)


@pytest.mark.parametrize("case", ["random", "reversed", "duplicate", "out_of_range", "keys_zero", "keys_max"])
def test_resort_any_earlier_order_gives_the_full_sort(case):
    s = synth.system(2)
    rng = np.random.default_rng(11)
    perm, keys = oracle.hilbert_sort(s.pos, s.box, 10)
    perm = perm.astype(np.int32)
    keys = keys.astype(np.uint32)
    if case == "random":
        perm = rng.permutation(s.n).astype(np.int32)
        keys = np.sort(rng.integers(0, 1 << 30, s.n)).astype(np.uint32)
    elif case == "reversed":
        perm, keys = perm[::-1].copy(), keys[::-1].copy()
    elif case == "duplicate":
        perm[5] = perm[6]
    elif case == "out_of_range":
        perm[100] = s.n + 7
        perm[200] = -3
    elif case == "keys_zero":
        keys[:] = 0
    elif case == "keys_max":
        keys[:] = 0xFFFFFFFF
    fast = False
    _check(s.pos, s.box, perm, keys.view(np.int32), expect_fast=fast)


@pytest.mark.parametrize("n", [1, 2, 3, 257, 1025, 4097, 20011])
@pytest.mark.parametrize("bits", [1, 2, 5, 10])
def test_resort_small_ragged_and_tied(n, bits):
    """Coarse grids put many atoms on one key: ties are decided by index
    in both paths."""
    rng = np.random.default_rng(n * 16 + bits)
    box = (23.0, 17.5, 31.25)
    pos0 = (rng.random((n, 3)) * np.array(box)).astype(np.float32)
    pos0 = _wrap(pos0.astype(np.float64), box)
    perm, keys = oracle.hilbert_sort(pos0, box, bits)
    pos1 = _wrap(pos0.astype(np.float64) + rng.normal(0, 0.05, pos0.shape), box)
    _check(pos1, box, perm.astype(np.int32), keys.astype(np.uint32).view(np.int32), bits=bits)


def test_resort_full_size_after_a_rebuild_interval():
    """10.24M atoms moved by 20 steps of 0.01 A per axis: incremental path,
    exact against the oracle's full sort."""
    s = synth.system(4)
    perm, keys = oracle.hilbert_sort(s.pos, s.box, 10)
    rng = np.random.default_rng(5)
    pos1 = _wrap(s.pos64 + rng.normal(0, 0.01 * np.sqrt(20), s.pos64.shape), s.box)
    _check(pos1, s.box, perm.astype(np.int32), keys.astype(np.uint32).view(np.int32), expect_fast=True)
