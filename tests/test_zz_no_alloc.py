"""The allocation-free Hilbert sort, tess_hilbert_sort_static.

Callers that cannot allocate device memory -- a plugin whose host program
owns every device buffer, or a time-step loop that must not call cudaMalloc
because it synchronises the device -- and that have no buffer to lend as a
workspace use this entry point.  Its scratch is an array inside the library,
shared by every call on a device, so the test checks that two calls in a row
(of different sizes, the second after the first has filled the array) give
exactly the permutation, keys and sorted positions of the workspace entry
point.  It goes through the C ABI, as a user of the library would.

This file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest

pytestmark = pytest.mark.gpu


def _call_static(tess, torch, pos, box, bits=10):
    n = pos.shape[0]
    dev = pos.device
    perm = torch.full((n,), -7, dtype=torch.int32, device=dev)
    keys = torch.zeros(n, dtype=torch.int32, device=dev)
    ps = torch.full((n, 4), float("nan"), dtype=torch.float32, device=dev)
    st = torch.full((1,), -1, dtype=torch.int32, device=dev)
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    code = tess.tess_hilbert_sort_static(P(pos), n, box, bits, P(perm), P(keys), P(ps), P(st), stream)
    assert code == 0, tess.tess_status_string(code)
    torch.cuda.synchronize()
    return perm.cpu().numpy(), keys.cpu().numpy(), ps.cpu().numpy(), int(st.item())


def _call_workspace(tess, torch, pos, box, bits=10):
    perm, keys, ps, st = tess.hilbert_sort(pos, box, bits)
    torch.cuda.synchronize()
    return perm.cpu().numpy(), keys.cpu().numpy(), ps.cpu().numpy(), int(st.item())


def test_static_sort_matches_workspace_sort_on_consecutive_calls():
    import torch
    import space_filling_curve_b200 as tess
    import synth

    assert torch.cuda.is_available()
    big = synth.system(2)                       # 98,304 atoms: fills a good part of the array
    small = synth.system(1)                     # 3,000 atoms: runs on what the first call left
    for s in (big, small):
        pos = torch.from_numpy(s.pos).cuda()
        got = _call_static(tess, torch, pos, s.box)
        want = _call_workspace(tess, torch, pos, s.box)
        assert got[3] == 0 and want[3] == 0
        assert np.array_equal(got[0], want[0]), "permutation differs"
        assert np.array_equal(got[1], want[1]), "keys differ"
        assert np.array_equal(got[2], want[2]), "sorted positions differ"


def test_static_sort_largest_size_and_limit():
    import torch
    import space_filling_curve_b200 as tess

    n = tess.HILBERT_SORT_STATIC_MAX_N
    rng = np.random.default_rng(11)
    box = (100.0, 100.0, 100.0)
    pos = torch.from_numpy((rng.uniform(0, 100.0, (n, 3))).astype(np.float32)).cuda()
    got = _call_static(tess, torch, pos, box)
    want = _call_workspace(tess, torch, pos, box)
    assert np.array_equal(got[0], want[0]) and np.array_equal(got[1], want[1])
    # one atom more than the array holds: refused before any launch
    P = ctypes.c_void_p(pos.data_ptr())
    code = tess.tess_hilbert_sort_static(P, n + 1, box, 10, P, None, None, None, None)
    assert code == 5 and "static scratch" in tess.tess_status_string(code)
