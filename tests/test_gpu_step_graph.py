"""The step graph (tess_step_graph_*): one time step as a CUDA graph whose
rebuild branch is a conditional node decided on the device.  Along a
trajectory it must take exactly the rebuild decisions, and produce exactly
the permutation, list and aggregation, of the same steps driven from the
host one call at a time; its decisions, orders and lists must match the
oracle, its aggregation within the aggregation's tolerance."""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import agg_error, canon_rows, torch_cuda

pytestmark = pytest.mark.gpu


def test_step_graph_along_a_trajectory():
    torch = torch_cuda()
    import space_filling_curve_b200 as tess
    s = synth.system(2)
    dev = torch.device("cuda", 0)
    frames = [s.pos] + [p for _, p in s.trajectory(40)]
    feat = torch.from_numpy(s.features()).to(dev)
    g = tess.StepGraph(torch.from_numpy(s.pos).to(dev), s.box, s.rc, s.skin, s.cap, feat)
    ref = None            # eager mirror: reference positions (sorted order, float4)
    perm = None
    decisions = []
    try:
        for t, p in enumerate(frames):
            pos = torch.from_numpy(p).to(dev)
            with torch.cuda.stream(g.stream):
                g.pos.copy_(pos)
                g.launch()
            g.stream.synchronize()
            # host-driven mirror with the same entry points
            if perm is None:
                rebuild = 1
            else:
                cur = torch.zeros((s.n, 4), dtype=torch.float32, device=dev)
                cur[:, :3] = pos[perm.long()]
                flag, _ = tess.skin_check(cur, ref, s.box, s.skin)
                rebuild = int(flag.item())
                # the oracle's decision on the same fp32 values
                assert rebuild == oracle.skin_check(cur.cpu().numpy(), ref.cpu().numpy(), s.box, s.skin)[0]
            if rebuild:
                perm, _, ref, _ = tess.hilbert_sort(pos, s.box)
                nbr, cnt, ov = tess.build_neighbors(ref, s.box, s.rc, s.skin, s.cap)
                cur = ref.clone()
            out = tess.edge_aggregate(cur, s.box, s.rc, nbr, cnt, feat)
            torch.cuda.synchronize()
            assert int(g.rebuild.item()) == rebuild
            assert torch.equal(g.perm, perm)
            assert torch.equal(g.counts, cnt)
            assert np.array_equal(canon_rows(g.nbr.cpu().numpy(), g.counts.cpu().numpy()),
                                  canon_rows(nbr.cpu().numpy(), cnt.cpu().numpy()))
            assert torch.equal(g.out, out)
            decisions.append(rebuild)
        assert decisions[0] == 1 and sum(decisions[1:]) >= 1
        assert g.rebuilds == sum(decisions)
        # the last state against the oracle
        last = max(i for i, d in enumerate(decisions) if d)
        want_perm, _ = oracle.hilbert_sort(frames[last], s.box, 10)
        assert np.array_equal(g.perm.cpu().numpy(), want_perm)
        ps = g.pos_sorted.cpu().numpy()
        onbr, ocnt, _ = oracle.neighbors_cells(ps, s.box, s.rc, s.skin, s.cap)
        assert np.array_equal(g.counts.cpu().numpy(), ocnt)
        assert np.array_equal(canon_rows(g.nbr.cpu().numpy(), ocnt), canon_rows(onbr, ocnt))
        cur = g.pos_cur.cpu().numpy()
        err, _ = agg_error(g.out.cpu().numpy(), oracle.edge_aggregate(cur, s.box, s.rc, onbr, ocnt, s.features()))
        assert err <= 1e-5
    finally:
        g.close()


def test_step_graph_forced_rebuild():
    torch = torch_cuda()
    import space_filling_curve_b200 as tess
    s = synth.system(1)
    dev = torch.device("cuda", 0)
    feat = torch.from_numpy(s.features()).to(dev)
    g = tess.StepGraph(torch.from_numpy(s.pos).to(dev), s.box, s.rc, s.skin, s.cap, feat)
    try:
        for _ in range(3):
            g.launch()
        g.request_rebuild()
        g.launch()
        g.stream.synchronize()
        assert int(g.rebuild.item()) == 1
        assert g.rebuilds == 2          # the first launch and the requested one
    finally:
        g.close()
