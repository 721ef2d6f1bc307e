"""The incremental re-sort's method, restated in numpy and checked against a
full sort (host logic; the CUDA kernels are checked in test_gpu_resort.py).

An element is "local" when its new key lies within the old keys of its
+-W old neighbors; local elements can then be out of order only with
elements at most 2W old ranks away, so two phases of block sorts of 4W
elements (the second offset by 2W) order them, and the others merge in by
rank.  Keys move like a trajectory (small steps, a few long jumps)."""
import numpy as np
import pytest

W = 64
D = 2 * W


def _block_sort(x, phase):
    x = x.copy()
    if phase == 0:
        for a in range(0, len(x), 2 * D):
            x[a:a + 2 * D] = np.sort(x[a:a + 2 * D])
    else:
        for a in range(D, len(x), 2 * D):
            x[a:a + 2 * D] = np.sort(x[a:a + 2 * D])
    return x


def _resort(old_keys, new_keys_in_old_order, idx_in_old_order):
    n = len(old_keys)
    k = np.arange(n)
    lo = old_keys[np.maximum(k - W, 0)]
    hi = old_keys[np.minimum(k + W, n - 1)]
    elem = (new_keys_in_old_order.astype(np.int64) << 32) | idx_in_old_order
    local = (new_keys_in_old_order >= lo) & (new_keys_in_old_order <= hi)
    S = _block_sort(_block_sort(elem[local], 0), 1)
    if len(S) > 1 and not np.all(S[1:] > S[:-1]):
        return None                                   # the device would fall back
    O = np.sort(elem[~local])
    out = np.empty(n, np.int64)
    out[np.arange(len(S)) + np.searchsorted(O, S)] = S
    out[np.arange(len(O)) + np.searchsorted(S, O)] = O
    return out


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
@pytest.mark.parametrize("n", [1, 7, 300, 5000, 40000])
def test_scheme_reproduces_the_full_sort(n, seed):
    rng = np.random.default_rng(seed * 100 + n % 97)
    idx0 = np.arange(n, dtype=np.int64)
    key0 = rng.integers(0, 1 << 30, n)
    order = np.lexsort((idx0, key0))                   # previous sort: by (key, index)
    old_keys = key0[order]
    # new keys, in the previous order: small moves for most, jumps for a few,
    # and some exact ties
    new = old_keys + rng.integers(-3000, 3000, n)
    jump = rng.random(n) < 0.01
    new[jump] = rng.integers(0, 1 << 30, int(jump.sum()))
    tie = rng.random(n) < 0.02
    new[tie] = new[np.maximum(np.arange(n)[tie] - 1, 0)]
    new = np.clip(new, 0, (1 << 30) - 1)
    got = _resort(old_keys, new, order)
    want_order = np.lexsort((order, new))
    want = (new[want_order].astype(np.int64) << 32) | order[want_order]
    assert got is not None                             # no fallback on trajectory-like moves
    assert np.array_equal(got, want)
