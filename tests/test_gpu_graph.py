"""The per-step path replayed as one CUDA graph (Tessera replays each
interval between rebuilds as a single CUDA graph; Tessera, abstract): every entry point
is stream-ordered, allocates nothing and never synchronises the host, so a
whole step -- sort, list, skin check, aggregation -- can be captured once and
replayed.  Replays must reproduce the eager results exactly (the kernels are
deterministic)."""
import numpy as np
import pytest

import synth
from gpu_util import torch_cuda

pytestmark = pytest.mark.gpu


def test_captured_step_replays_exactly():
    torch = torch_cuda()
    import space_filling_curve_b200 as tess
    s = synth.system(2)
    dev = torch.device("cuda", 0)
    n, cap, F = s.n, s.cap, s.F
    pos = torch.from_numpy(s.pos).to(dev)
    nxt = torch.from_numpy(next(iter(s.trajectory(1)))[1]).to(dev)
    ws_s = torch.empty(tess.tess_hilbert_sort_workspace(n), dtype=torch.uint8, device=dev)
    ws_n = torch.empty(tess.tess_build_neighbors_workspace(n, s.box, s.rc, s.skin), dtype=torch.uint8, device=dev)
    perm = torch.empty(n, dtype=torch.int32, device=dev)
    keys = torch.empty(n, dtype=torch.int32, device=dev)
    ps = torch.empty((n, 4), dtype=torch.float32, device=dev)
    st = torch.empty(1, dtype=torch.int32, device=dev)
    nbr = torch.empty((n, cap), dtype=torch.int32, device=dev)
    cnt = torch.empty(n, dtype=torch.int32, device=dev)
    ov = torch.empty(1, dtype=torch.int32, device=dev)
    cur = torch.zeros((n, 4), dtype=torch.float32, device=dev)
    rb = torch.empty(1, dtype=torch.int32, device=dev)
    md = torch.empty(1, dtype=torch.float64, device=dev)
    feat = torch.randn((n, F), generator=torch.Generator(device=dev).manual_seed(1), device=dev)
    out = torch.empty((n, F), dtype=torch.float32, device=dev)

    def step():
        tess.hilbert_sort(pos, s.box, ws=ws_s, perm=perm, keys_sorted=keys, pos_sorted=ps, dev_status=st)
        tess.build_neighbors(ps, s.box, s.rc, s.skin, cap, ws=ws_n, nbr=nbr, counts=cnt, overflow=ov)
        tess.skin_check(cur, ps, s.box, s.skin, rebuild=rb, max_disp2=md)
        tess.edge_aggregate(ps, s.box, s.rc, nbr, cnt, feat, out=out)

    step()
    torch.cuda.synchronize()
    cur[:, :3] = nxt[perm.long()]
    step()
    torch.cuda.synchronize()
    eager = [t.clone() for t in (perm, ps, nbr, cnt, ov, rb, md, out)]

    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()                       # warm the side stream before capture
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        step()
    for t in (perm, ps, nbr, cnt, out):
        t.zero_()
    for _ in range(2):
        g.replay()
        torch.cuda.synchronize()
        for a, b in zip(eager, (perm, ps, nbr, cnt, ov, rb, md, out)):
            assert torch.equal(a, b)
