"""Benchmark of the neighbor-rebuild hot path on B200.

One step = one full neighbor rebuild of the 10.24M-atom salt solution
(rc 5.75 A, skin 0.5 A, 160 neighbors per row):
    Hilbert sort -> padded neighbor list
with every input resident in HBM when the timed region starts.  The value is
atoms per second over all ranks (weak scaling: with --gpus N each rank runs
an independent replica of the same workload, there is no collective in the
data path).  The line also carries the whole step (rebuild, skin check,
aggregation of 64 features), the end-to-end rate with host copies, and with
--all-configs the same figures for all five workloads.

Prints one JSON line (rank 0).  ``--impl reference`` times the CPU oracle
instead (a deliberately plain program, on the host cores, on a bounded
sample of the workload).
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "atoms/s for full neighbor rebuild at 10.24M atoms (1 B200); % of HBM roofline"
WORKLOAD_CFG = 4


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi clock samples during the timed region."""

    def __init__(self, index: int):
        self.index = index
        self.samples = []
        self._stop = threading.Event()
        self._proc = None

    def __enter__(self):
        q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")
        try:
            self._proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), "--query-gpu=" + q,
                                           "--format=csv,noheader,nounits", "-lms", "50"],
                                          stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except (OSError, FileNotFoundError):
            self._proc = None
        return self

    def running(self):
        return self._proc is not None and self._proc.poll() is None

    def mark(self):
        """Start of the timed region: drop the samples taken so far (the
        sampler is started earlier, during the warm-up, because nvidia-smi
        can take a while to print its first line)."""
        self.samples.clear()

    def _read(self):
        for line in self._proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 7:
                self.samples.append(parts)

    def __exit__(self, *a):
        if self._proc is not None:
            self._proc.terminate()
            try:
                self._proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self._proc.kill()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(s[0]) for s in self.samples if s[0].replace(".", "").isdigit()]
        mx = [float(s[1]) for s in self.samples if s[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for s in self.samples for k in range(4) if s[3 + k].lower() == "active"})
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.samples)}


def _dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a per-rank float over all ranks (identity for one rank)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, world: int, device=None) -> float:
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ---------------------------------------------------------------- CUDA arm


class Step:
    """All device buffers of one replica, and the path through the C ABI."""

    def __init__(self, s, device, pad_fill=True, search="default", curve="hilbert"):
        import torch
        import space_filling_curve_b200 as tess
        self.tess = tess
        self.s = s
        self.n = s.n
        self.box = s.box
        self.dev = device
        n, cap, F = s.n, s.cap, s.F
        self.pos3 = torch.from_numpy(s.pos).to(device)
        self.ws_sort = torch.empty(tess.tess_hilbert_sort_workspace(n), dtype=torch.uint8, device=device)
        self.ws_nbr = torch.empty(tess.tess_build_neighbors_workspace(n, s.box, s.rc, s.skin), dtype=torch.uint8,
                                  device=device)
        self.perm = torch.empty(n, dtype=torch.int32, device=device)
        self.keys = torch.empty(n, dtype=torch.int32, device=device)
        self.pos_sorted = torch.empty((n, 4), dtype=torch.float32, device=device)
        self.status = torch.empty(1, dtype=torch.int32, device=device)
        self.nbr = torch.empty((n, cap), dtype=torch.int32, device=device)
        self.counts = torch.empty(n, dtype=torch.int32, device=device)
        self.overflow = torch.empty(1, dtype=torch.int32, device=device)
        self.rebuild_flag = torch.empty(1, dtype=torch.int32, device=device)
        self.maxd = torch.empty(1, dtype=torch.float64, device=device)
        g = torch.Generator(device=device)
        g.manual_seed(s.seed)
        # features live in the sorted index space (produced there by the model)
        self.feat = torch.randn((n, F), generator=g, device=device, dtype=torch.float32)
        self.out = torch.empty((n, F), dtype=torch.float32, device=device)
        self.flags = (0 if pad_fill else tess.TESS_NO_PAD_FILL) | tess.SEARCH_FLAGS[search]
        # curve "none": no sort at all; the atoms stay in a fixed random order
        # (the locality baseline: what the list and the aggregation cost
        # without a space-filling-curve order)
        self.sort_fn = {"hilbert": tess.tess_hilbert_sort, "morton": tess.tess_morton_sort, "none": None}[curve]
        if self.sort_fn is None:
            shuffle = torch.randperm(n, generator=torch.Generator().manual_seed(s.seed)).to(device)
            self.perm.copy_(shuffle.int())
            self.pos_sorted.zero_()
            self.pos_sorted[:, :3] = self.pos3[shuffle]
        # the next frame of the trajectory, in the sorted order of frame 0
        t1 = next(iter(s.trajectory(1, condition=False)))[1]
        self.frame1 = torch.from_numpy(t1).to(device)
        self.pos_next = torch.empty((n, 4), dtype=torch.float32, device=device)
        self.run()
        torch.cuda.synchronize()
        self.pos_next.zero_()
        self.pos_next[:, :3] = self.frame1[self.perm.long()]
        torch.cuda.synchronize()

    @staticmethod
    def _ptr(t):
        import ctypes
        return ctypes.c_void_p(t.data_ptr())

    def _stream(self):
        import ctypes
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    def rebuild(self, pos3=None, perm=None, counts=None, overflow=None, status=None):
        """The timed unit: Hilbert sort, then the padded neighbor list.  The
        outputs a caller copies out (perm, counts, the two status words) may
        be given as other buffers."""
        tess, s, P, st = self.tess, self.s, self._ptr, self._stream()
        pos3 = self.pos3 if pos3 is None else pos3
        perm = self.perm if perm is None else perm
        counts = self.counts if counts is None else counts
        overflow = self.overflow if overflow is None else overflow
        status = self.status if status is None else status
        if self.sort_fn is not None:
            c = self.sort_fn(P(pos3), self.n, s.box, 10, P(self.ws_sort), self.ws_sort.numel(),
                             P(perm), P(self.keys), P(self.pos_sorted), P(status), st)
            assert c == 0, c
        c = tess.tess_build_neighbors(P(self.pos_sorted), self.n, s.box, s.rc, s.skin, s.cap, self.flags,
                                      P(self.ws_nbr), self.ws_nbr.numel(), P(self.nbr), P(counts),
                                      P(overflow), st)
        assert c == 0, c

    def per_step(self):
        """What every MD step runs between rebuilds: skin check, aggregation."""
        tess, s, P, st = self.tess, self.s, self._ptr, self._stream()
        c = tess.tess_skin_check(P(self.pos_next), P(self.pos_sorted), self.n, s.box, s.skin,
                                 P(self.rebuild_flag), P(self.maxd), st)
        assert c == 0, c
        c = tess.tess_edge_aggregate(P(self.pos_sorted), self.n, s.box, s.rc, P(self.nbr), P(self.counts), s.cap,
                                     P(self.feat), s.F, P(self.out), None, None, None, st)
        assert c == 0, c

    def run(self, pos3=None):
        """The whole path once: rebuild, skin check, aggregation."""
        self.rebuild(pos3)
        self.per_step()


def _algorithmic_bytes(n, mean_count, F):
    """Minimum bytes each stage must move per launch (the per-atom figures of
    the design notes times n)."""
    return {
        "hilbert_keys": n * (16 + 8),
        "key_sort": n * (12 + 36),          # the ideal single pass plus the fused gather of perm / positions
        "cell_binning": n * 28,
        "pair_search": n * (16 + 4 * mean_count + 4),
        "skin_check": n * 32,
        "edge_aggregate": n * (4 * F + 4 * F + 16 + 4 * mean_count + 4),
    }


def rebuild_bytes(n, mean_count):
    """Algorithmic bytes of one full rebuild: keys 24, sort 12, gather 36,
    binning 28, pair search 16 + 4 * mean count + 4 (per atom)."""
    return n * (24 + 12 + 36 + 28 + 16 + 4 * mean_count + 4)


def _timed(fn, steps, flush):
    """Per-call CUDA events on the current stream around fn(); the 256 MB
    flush write runs before each call, outside its events.  Returns the list
    of per-call milliseconds."""
    import torch
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for k in range(steps):
        flush.zero_()
        evs[k][0].record()
        fn()
        evs[k][1].record()
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


def _stage_ms(stages):
    return {k: v[0] / v[1] for k, v in stages.items() if v[1] > 0}


def _config_summary(step, steps, flush, peak):
    """Rebuild, skin check and aggregation of one workload, each timed alone
    (stage timing on; per-call means)."""
    import torch
    tess, s = step.tess, step.s
    tess.tess_stage_times()
    tess.tess_stage_timing(True)
    reb = _timed(step.rebuild, steps, flush)
    per = _timed(step.per_step, steps, flush)
    tess.tess_stage_timing(False)
    st = _stage_ms(tess.tess_stage_times())
    counts = step.counts.double()
    mean = float(counts.mean().item())
    pairs = float(counts.sum().item())
    n = s.n
    rb = rebuild_bytes(n, mean)
    ab = _algorithmic_bytes(n, mean, s.F)
    reb_ms = sum(reb) / len(reb)
    out = {
        "workload": s.name, "atoms": n, "box": list(s.box), "rc": s.rc, "skin": s.skin, "cap": s.cap, "F": s.F,
        "mean_neighbors": mean, "overflow": int(step.overflow.item()),
        "rebuild_ms": reb_ms, "rebuild_atoms_per_s": n / (reb_ms / 1e3), "pairs_per_s": pairs / (reb_ms / 1e3),
        "rebuild_frac_hbm": rb / (reb_ms / 1e3) / 1e9 / peak,
        "stages_ms": {k: round(v, 4) for k, v in st.items()},
    }
    if "pair_search" in st:
        out["pair_search_frac_hbm"] = ab["pair_search"] / (st["pair_search"] / 1e3) / 1e9 / peak
    if "skin_check" in st:
        out["skin_check_gbs"] = ab["skin_check"] / (st["skin_check"] / 1e3) / 1e9
        out["skin_check_atoms_per_s"] = n / (st["skin_check"] / 1e3)
    if "edge_aggregate" in st:
        out["aggregate_gbs"] = ab["edge_aggregate"] / (st["edge_aggregate"] / 1e3) / 1e9
        out["aggregate_frac_hbm"] = out["aggregate_gbs"] / peak
        out["aggregate_pairs_per_s"] = pairs / (st["edge_aggregate"] / 1e3)
    del torch
    return out


def run_cuda(args, world, rank, local):
    import torch
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    import synth
    import space_filling_curve_b200 as tess
    s = synth.system(args.config)
    step = Step(s, dev, pad_fill=not args.no_pad_fill, search=args.search, curve=args.curve)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    peak, peak_kind = _peaks()

    # clocks: the sampler starts with the warm-up and keeps the samples from
    # the timed rebuilds and the timed loops right after them (same load)
    clk = ClockSampler(local).__enter__()
    # warm-up (W whole steps); stage timing on so that its event pool fills
    tess.tess_stage_times()
    tess.tess_stage_timing(True)
    for _ in range(args.warmup):
        flush.zero_()
        step.run()
    torch.cuda.synchronize()
    tess.tess_stage_times()
    ov = int(step.overflow.item())
    counts = step.counts.double()
    mean_count = float(counts.mean().item())
    pairs = float(counts.sum().item())

    # timed region: K rebuilds (sort + list), per-rebuild events on the
    # launching stream, L2 flushed before each, the library's stage timing off
    tess.tess_stage_timing(False)
    # keep the GPU busy until the clock sampler has printed (at most ~3 s more)
    extra = 0
    while clk.running() and not clk.samples and extra < 600:
        step.rebuild()
        torch.cuda.synchronize()
        extra += 1
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    launches0 = tess.tess_kernel_launch_count()
    clk.mark()
    reb = _timed(step.rebuild, args.steps, flush)
    if world > 1:
        torch.distributed.barrier()
    launches = tess.tess_kernel_launch_count() - launches0
    ms = sum(reb)
    ms_max = max_over_ranks(ms, world, dev)
    n_total = sum_over_ranks(float(s.n * args.steps), world, dev)
    value = n_total / (ms_max / 1e3)

    # a separate pass of the same rebuilds with the library's stage events
    # (pooled, no event creation) for the per-kernel durations
    tess.tess_stage_timing(True)
    tess.tess_stage_times()
    staged_ms = sum(_timed(step.rebuild, args.steps, flush)) / args.steps
    stage_ms = _stage_ms(tess.tess_stage_times())
    tess.tess_stage_timing(False)

    # the whole step (rebuild + skin check + aggregation), for context
    tess.tess_stage_timing(True)
    whole = _timed(step.run, args.steps, flush)
    whole_stages = _stage_ms(tess.tess_stage_times())
    tess.tess_stage_timing(False)
    whole_ms = sum(whole) / args.steps
    clk.__exit__(None, None, None)

    extras = _extras(args, step, flush, dev, world, ms_max)

    # e2e: through the C ABI with host buffers (pinned); every rebuild's
    # copies (positions in; perm, counts and the status words out -- the list
    # itself stays on the device for the steps that use it) are inside the
    # timed region, issued on two copy streams (one per direction) with double
    # buffers so that they overlap the neighboring rebuilds and each other, as
    # a stream-ordered caller would
    e2e_val, e2e_steps = _e2e(step, s, args.steps, world, dev)

    nbytes = _algorithmic_bytes(s.n, mean_count, s.F)
    ps_ms = stage_ms.get("pair_search")
    achieved = nbytes["pair_search"] / (ps_ms / 1e3) / 1e9 if ps_ms else None
    rb = rebuild_bytes(s.n, mean_count)
    reb_ms = ms_max / args.steps
    traffic = _traffic_from_profile("pair_search", s.n, s.name)
    clocks = clk.summary()

    all_cfg = None
    if args.all_configs:
        all_cfg = []
        for cfg in (1, 2, 3, 4, 5):
            sc = s if cfg == args.config else synth.system(cfg)
            stc = step if cfg == args.config else Step(sc, dev, pad_fill=not args.no_pad_fill,
                                                       search=args.search, curve=args.curve)
            all_cfg.append(_config_summary(stc, max(3, args.steps), flush, peak))
            if stc is not step:
                del stc
                torch.cuda.empty_cache()

    if rank == 0:
        line = {
            "metric": METRIC,
            "value": value,
            "unit": "atoms/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": reb_ms,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "f32",
            "data": "synthetic (seeded salt-solution generator; no dataset)",
            "config": {
                "workload": "%s: %d atoms, box %.3f x %.3f x %.3f A, rc %.2f, skin %.2f, cap %d; step = full "
                            "neighbor rebuild: hilbert_sort + build_neighbors (pad-filled list)"
                            % (s.name, s.n, s.box[0], s.box[1], s.box[2], s.rc, s.skin, s.cap),
                "atoms": s.n,
                "pad_fill": not args.no_pad_fill,
                "pair_search": args.search, "library": tess.tess_version(),
                "curve": args.curve,
                "l2": "flushed before every timed rebuild (256 MB write, outside its events)",
                "parallelism": "replicas (no collective in the data path)",
                "mean_neighbors": mean_count,
                "pairs_listed": pairs,
                "overflow": ov,
            },
            "stages_ms": {k: round(v, 4) for k, v in stage_ms.items()},
            "rebuild_ms_stage_timing_on": staged_ms,
            "pairs_per_s": pairs / (reb_ms / 1e3),
            "roofline": {
                "bound": "hbm",
                "kernel": "pair_search",
                "achieved": achieved,
                "peak": peak,
                "peak_kind": peak_kind,
                "unit": "GB/s",
                "frac": achieved / peak if achieved else None,
                "traffic": traffic,
                "algorithmic_bytes": nbytes["pair_search"],
                "ms": ps_ms,
            },
            "rebuild_roofline": {
                "bound": "hbm", "ms": reb_ms, "algorithmic_bytes": rb,
                "achieved": rb / (reb_ms / 1e3) / 1e9, "peak": peak, "unit": "GB/s",
                "frac": rb / (reb_ms / 1e3) / 1e9 / peak,
            },
            "step": {"what": "rebuild + skin check + edge aggregate (F %d)" % s.F, "ms": whole_ms,
                     "atoms_per_s": s.n / (whole_ms / 1e3),
                     "stages_ms": {k: round(v, 4) for k, v in whole_stages.items()}},
            "e2e": {"value": e2e_val, "unit": "atoms/s", "steps": e2e_steps, "pipelined": True,
                    "h2d_bytes_per_step": s.n * 12, "d2h_bytes_per_step": s.n * 8 + 8,
                    "note": "positions in; perm, counts and status words out; the list stays on the device"},
            "gpu_launches": launches,
            "clocks": clocks,
        }
        line.update(extras)
        if all_cfg is not None:
            line["all_configs"] = all_cfg
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(args)
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


def _e2e(step, s, steps, world, dev):
    import torch
    host_pos = torch.from_numpy(s.pos).pin_memory()
    host_perm = [torch.empty(s.n, dtype=torch.int32).pin_memory() for _ in range(2)]
    host_counts = [torch.empty(s.n, dtype=torch.int32).pin_memory() for _ in range(2)]
    host_flags = [torch.empty(2, dtype=torch.int32).pin_memory() for _ in range(2)]
    pos_in = [torch.empty_like(step.pos3) for _ in range(2)]
    st_perm = [torch.empty_like(step.perm) for _ in range(2)]
    st_counts = [torch.empty_like(step.counts) for _ in range(2)]
    st_flags = [torch.empty(2, dtype=torch.int32, device=dev) for _ in range(2)]
    cs = torch.cuda.current_stream()
    xs = torch.cuda.Stream(device=dev)       # host -> device copies
    ys = torch.cuda.Stream(device=dev)       # device -> host copies (the other direction of the link)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    ev_read = [torch.cuda.Event() for _ in range(2)]
    # at least 30 rebuilds, so that filling and draining the copy pipeline
    # (the first positions in, the last results out) weighs as in a long run
    e2e_steps = max(30, steps)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(cs)
    xs.wait_stream(cs)
    with torch.cuda.stream(xs):
        for b in range(min(2, e2e_steps)):
            pos_in[b].copy_(host_pos, non_blocking=True)
            ev_in[b].record(xs)
    for t in range(e2e_steps):
        b = t % 2
        cs.wait_event(ev_in[b])
        if t >= 2:
            cs.wait_event(ev_read[b])            # rebuild t-2's results have left output buffer set b
        # the rebuild writes its perm, counts and status words straight into buffer set b
        step.rebuild(pos3=pos_in[b], perm=st_perm[b], counts=st_counts[b], overflow=st_flags[b][0:1],
                     status=st_flags[b][1:2])
        ev_out[b].record(cs)
        with torch.cuda.stream(ys):
            ys.wait_event(ev_out[b])
            host_perm[b].copy_(st_perm[b], non_blocking=True)
            host_counts[b].copy_(st_counts[b], non_blocking=True)
            host_flags[b].copy_(st_flags[b], non_blocking=True)
            ev_read[b].record(ys)
        if t + 2 < e2e_steps:                      # rebuild t has read pos_in[b]: load t+2's positions
            with torch.cuda.stream(xs):
                xs.wait_event(ev_out[b])
                pos_in[b].copy_(host_pos, non_blocking=True)
                ev_in[b].record(xs)
    cs.wait_stream(xs)
    cs.wait_stream(ys)
    e1.record(cs)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    return sum_over_ranks(float(s.n * e2e_steps), world, dev) / (e2e_ms / 1e3), e2e_steps


def _extras(args, step, flush, dev, world, rebuild_ms_total):
    """The optional measurements (--backward, --resort, --monitor,
    --step-graph, --graph); each returns a dict under its own key."""
    import ctypes
    import torch
    tess, s = step.tess, step.s
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    stc = lambda: ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    out = {}

    def mean_ms(call):
        for _ in range(args.warmup):
            assert call() == 0
        return sum(_timed(call, args.steps, flush)) / args.steps

    if args.backward:
        # the aggregation's backward (force path) on the same list, timed alone
        gout = torch.randn((s.n, s.F), generator=torch.Generator(device=dev).manual_seed(2), device=dev)
        gfeat = torch.empty_like(gout)
        gpos = torch.empty((s.n, 3), dtype=torch.float32, device=dev)
        mean_count = float(step.counts.double().mean().item())
        bms = mean_ms(lambda: tess.tess_edge_aggregate_backward(P(step.pos_sorted), s.n, s.box, s.rc, P(step.nbr),
                                                                P(step.counts), s.cap, P(step.feat), P(gout), s.F,
                                                                P(gfeat), P(gpos), stc()))
        bbytes = s.n * (3 * 4 * s.F + 16 + 4 * mean_count + 4 + 12)
        out["backward"] = {"ms": bms, "algorithmic_bytes": bbytes, "achieved_gbs": bbytes / (bms / 1e3) / 1e9}

    if args.resort:
        # the re-sort at the next rebuild: every atom moved by a rebuild
        # interval of the trajectory's random walk (20 steps of sigma per axis)
        L = torch.tensor(s.box, dtype=torch.float64, device=dev)
        x = step.pos3.double() + torch.randn(step.pos3.shape, generator=torch.Generator(device=dev).manual_seed(4),
                                             device=dev, dtype=torch.float64) * (s.sigma * 20 ** 0.5)
        pos1 = (x - L * torch.floor(x / L)).float()
        pos1 = torch.where(pos1 >= L.float(), torch.zeros_like(pos1), pos1).contiguous()
        perm0, keys0 = step.perm.clone(), step.keys.clone()
        ws_rs = torch.empty(tess.tess_hilbert_resort_workspace(s.n), dtype=torch.uint8, device=dev)
        perm1 = torch.empty_like(perm0)
        keys1 = torch.empty_like(keys0)
        ps1 = torch.empty((s.n, 4), dtype=torch.float32, device=dev)
        st1 = torch.empty(1, dtype=torch.int32, device=dev)
        res = {"sigma_total": s.sigma * 20 ** 0.5}
        res["full_sort_ms"] = mean_ms(lambda: tess.tess_hilbert_sort(P(pos1), s.n, s.box, 10, P(step.ws_sort),
                                                                     step.ws_sort.numel(), P(perm1), P(keys1),
                                                                     P(ps1), P(st1), stc()))
        res["resort_ms"] = mean_ms(lambda: tess.tess_hilbert_resort(P(pos1), s.n, s.box, 10, P(perm0), P(keys0),
                                                                    P(ws_rs), ws_rs.numel(), P(perm1), P(keys1),
                                                                    P(ps1), P(st1), stc()))
        res["incremental_path"] = not (int(st1.item()) & tess.TESS_DEV_FULL_SORT)
        out["resort"] = res

    if args.monitor:
        # the closest listed pair on the step's list
        mws = torch.empty(tess.tess_min_pair_distance_workspace(), dtype=torch.uint8, device=dev)
        r2m = torch.empty(1, dtype=torch.float64, device=dev)
        pairm = torch.empty(2, dtype=torch.int32, device=dev)
        pairs = float(step.counts.double().sum().item())
        mms = mean_ms(lambda: tess.tess_min_pair_distance(P(step.pos_sorted), s.n, s.box, P(step.nbr), P(step.counts),
                                                          s.cap, P(mws), mws.numel(), P(r2m), P(pairm), stc()))
        out["min_pair"] = {"ms": mms, "min_distance": float(r2m.item()) ** 0.5, "pair": [int(v) for v in pairm.cpu()],
                           "list_bytes_read_gbs": pairs * 4 / (mms / 1e3) / 1e9}

    if args.step_graph:
        out["step_graph"] = _step_graph_loop(step, dev)

    if args.graph:
        # the whole step captured once as a CUDA graph and replayed
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            step.run()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        with torch.cuda.graph(g):
            step.run()
        for _ in range(args.warmup):
            flush.zero_()
            g.replay()
        torch.cuda.synchronize()
        gms = max_over_ranks(sum(_timed(g.replay, args.steps, flush)), world, dev)
        eager = max_over_ranks(sum(_timed(step.run, args.steps, flush)), world, dev)
        out["graph"] = {"ms_per_step": gms / args.steps, "eager_ms_per_step": eager / args.steps,
                        "speedup": eager / gms}
        del g
    return out


def _step_graph_loop(step, dev):
    """A time-step loop over a random walk (sigma per axis per step): the step
    graph decides rebuilds on the device; the eager loop reads the skin
    check's flag back every step and calls the rebuild itself."""
    import ctypes
    import torch
    tess, s = step.tess, step.s
    nsteps = 30
    gen = torch.Generator(device=dev).manual_seed(5)
    L = torch.tensor(s.box, dtype=torch.float32, device=dev)
    walk = [step.pos3.clone()]
    for _ in range(nsteps):
        x = walk[-1] + torch.randn(walk[-1].shape, generator=gen, device=dev) * s.sigma
        walk.append(torch.remainder(x, L).contiguous())
    sg = tess.StepGraph(walk[0], s.box, s.rc, s.skin, s.cap, step.feat)
    try:
        def run_graph():
            for t in range(nsteps):
                sg.pos.copy_(walk[t])
                sg.launch()
        with torch.cuda.stream(sg.stream):
            run_graph()                                    # warm-up (and first rebuild)
            sg.request_rebuild()
        before = sg.rebuilds
        with torch.cuda.stream(sg.stream):
            a_ev, b_ev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a_ev.record()
            run_graph()
            b_ev.record()
        sg.stream.synchronize()
        g_ms = a_ev.elapsed_time(b_ev) / nsteps
        g_rebuilds = sg.rebuilds - before
    finally:
        sg.close()
    ref4 = torch.empty((s.n, 4), dtype=torch.float32, device=dev)
    cur4 = torch.zeros((s.n, 4), dtype=torch.float32, device=dev)
    flag = torch.empty(1, dtype=torch.int32, device=dev)
    md2 = torch.empty(1, dtype=torch.float64, device=dev)
    P = lambda t_: ctypes.c_void_p(t_.data_ptr())
    stc = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    def run_eager():
        rebuilds = 0
        for t in range(nsteps):
            pos = walk[t]
            if t == 0:
                r = 1
            else:
                cur4[:, :3] = pos[step.perm.long()]
                assert tess.tess_skin_check(P(cur4), P(ref4), s.n, s.box, s.skin, P(flag), P(md2), stc) == 0
                r = int(flag.item())                     # the host round trip of a host-driven loop
            if r:
                rebuilds += 1
                assert step.sort_fn(P(pos), s.n, s.box, 10, P(step.ws_sort), step.ws_sort.numel(), P(step.perm),
                                    P(step.keys), P(ref4), P(step.status), stc) == 0
                assert tess.tess_build_neighbors(P(ref4), s.n, s.box, s.rc, s.skin, s.cap, 0, P(step.ws_nbr),
                                                 step.ws_nbr.numel(), P(step.nbr), P(step.counts),
                                                 P(step.overflow), stc) == 0
                cur4.copy_(ref4)
            assert tess.tess_edge_aggregate(P(cur4), s.n, s.box, s.rc, P(step.nbr), P(step.counts), s.cap,
                                            P(step.feat), s.F, P(step.out), None, None, None, stc) == 0
        return rebuilds
    run_eager()
    torch.cuda.synchronize()
    a_ev, b_ev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a_ev.record()
    e_rebuilds = run_eager()
    b_ev.record()
    torch.cuda.synchronize()
    e_ms = a_ev.elapsed_time(b_ev) / nsteps
    return {"steps": nsteps, "sigma": s.sigma, "graph_ms_per_step": g_ms, "eager_ms_per_step": e_ms,
            "speedup": e_ms / g_ms, "graph_rebuilds": g_rebuilds, "eager_rebuilds": e_rebuilds}


def _traffic_from_profile(kernel_stage, n, workload=""):
    """DRAM bytes per launch of the dominant kernel at n atoms, from the
    committed ncu summary (profiles/<stage>_traffic.json: bytes per atom of
    one capture), or None when there is none, when the kernel's source file
    has changed since the counters were taken, or when the workload is not
    of the captured family (bytes per atom depend on the neighbor counts)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "%s_traffic.json" % kernel_stage)
    try:
        with open(path) as f:
            d = json.load(f)
        with open(os.path.join(ROOT, d["source_file"]), "rb") as f:
            if hashlib.sha1(f.read()).hexdigest() != d["source_sha1"]:
                return None
        if not workload.startswith(d.get("workload_family", "")):
            return None
        return d["dram_bytes_per_atom"] * n
    except Exception:
        return None


# ---------------------------------------------------------------- oracle arm


def _oracle_step(s):
    """One full rebuild on the CPU oracle: Hilbert sort, then the cell-list
    Verlet list."""
    import oracle
    perm, keys, ps, nbr, cnt, ov = oracle.rebuild(s.pos, s.box, s.rc, s.skin, s.cap)
    return int(cnt.sum())


def _sample_system(budget_steps: int):
    """The bounded sample the oracle runs: the same salt-solution generator
    and parameters at 1.024M atoms (config 3), or 98k atoms (config 2) when
    many steps are asked for."""
    import synth
    return synth.system(3 if budget_steps <= 6 else 2)


def cpu_baseline(args):
    import oracle
    s = _sample_system(1)
    # repeated rebuilds of the sample for about 10 s of CPU work
    reps = 0
    t = time.perf_counter()
    while True:
        _oracle_step(s)
        reps += 1
        dt = time.perf_counter() - t
        if dt >= 10.0 or reps >= 100:
            break
    return {"value": s.n * reps / dt, "unit": "atoms/s", "cores": oracle.get_threads(), "kind": "oracle",
            "sample": "%d full rebuilds (Hilbert sort, cell-list Verlet list) of %s "
                      "(%d atoms, same generator and rc/skin/cap/F family as the 10.24M workload), %.1f s"
                      % (reps, s.name, s.n, dt)}


def run_reference(args, world, rank):
    if rank != 0:
        return
    import oracle
    s = _sample_system(args.steps + args.warmup)
    for _ in range(args.warmup):
        _oracle_step(s)
    t = time.perf_counter()
    for _ in range(args.steps):
        _oracle_step(s)
    dt = time.perf_counter() - t
    value = s.n * args.steps / dt
    sample = "%s (%d atoms) per rebuild, the plain CPU oracle on %d host threads" % (s.name, s.n, oracle.get_threads())
    line = {
        "impl": "reference",
        "metric": METRIC,
        "value": value,
        "unit": "atoms/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded salt-solution generator; no dataset)",
        "config": {"workload": "salt-10.24M (sampled: %s)" % s.name, "atoms": s.n},
        "cpu_baseline": {"value": value, "unit": "atoms/s", "cores": oracle.get_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "atoms/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["tess", "reference"], default="tess")
    ap.add_argument("--config", type=int, default=WORKLOAD_CFG)
    ap.add_argument("--no-pad-fill", action="store_true")
    ap.add_argument("--search", choices=["default", "tile", "lane", "lane2"], default="default",
                    help="pair search kernel (default: the library's choice)")
    ap.add_argument("--curve", choices=["hilbert", "morton", "none"], default="hilbert",
                    help="space-filling curve of the sort (morton: the comparison curve; none: no sort, atoms "
                         "in a fixed random order -- a locality baseline, not a rebuild)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--graph", action="store_true", help="also time the step captured as one CUDA graph")
    ap.add_argument("--backward", action="store_true", help="also time the aggregation's backward on the same list")
    ap.add_argument("--step-graph", action="store_true",
                    help="also time a 30-step loop as the device-decided step graph against a host-driven loop")
    ap.add_argument("--monitor", action="store_true", help="also time the closest-listed-pair check on the step's list")
    ap.add_argument("--resort", action="store_true",
                    help="also time the incremental re-sort against the full sort a rebuild interval later")
    ap.add_argument("--all-configs", action="store_true",
                    help="also report rebuild, skin check and aggregation on all five workloads")
    args = ap.parse_args(argv)
    world, rank, local = _dist_setup(args)
    if args.impl == "reference":
        run_reference(args, world, rank)
    else:
        run_cuda(args, world, rank, local)


if __name__ == "__main__":
    main()
