"""The sort's inter-block wait is bounded: when a predecessor tile never
publishes, the look-back gives up, sets TESS_DEV_TIMEOUT and the kernel
finishes, so the context stays usable (a fail-soft device condition, made
on purpose by tess_debug_lookback_timeout: no fault, no trap, no hang)."""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import torch_cuda

pytestmark = pytest.mark.gpu

TIMEOUT = 4


def test_lookback_wait_gives_up_and_reports():
    torch = torch_cuda()
    import ctypes
    import space_filling_curve_b200 as tess
    dev = torch.device("cuda", 0)
    ws = torch.empty(tess.tess_debug_lookback_timeout_workspace(), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    code = tess.tess_debug_lookback_timeout(ctypes.c_void_p(ws.data_ptr()), ws.numel(),
                                            ctypes.c_void_p(status.data_ptr()),
                                            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert code == 0
    torch.cuda.synchronize()
    assert int(status.item()) & TIMEOUT
    # the context is still usable: a normal sort right after is exact and clean
    s = synth.system(1)
    perm, keys, ps, st = tess.hilbert_sort(torch.from_numpy(s.pos).to(dev), s.box)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert np.array_equal(perm.cpu().numpy(), oracle.hilbert_sort(s.pos, s.box, 10)[0])
