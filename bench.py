#!/usr/bin/env python
"""Benchmark of the B200 selective-scan (S6) forward at the Mamba-130M layer
shape (batch 8, seqlen 2048, dim 1536, dstate 16, bf16 io, fp32 state).

One step = one forward selective scan over one batch of synthetic inputs (the
whole hot path: softplus, discretisation, recurrence, readout, D skip and
gate, fused in one kernel).  Prints one JSON line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Timing: inputs are resident in HBM; each step is bracketed by CUDA events on
the launching stream, and the L2 is flushed (a 256 MiB write) between steps,
outside the events.  The device time of the K steps is summed; under torchrun
every rank runs its own batch (weak scaling, no data-path collective) and
rank 0 reports the max over ranks.  `e2e` repeats the measurement through the
public binding with inputs copied from pinned host memory and the output
copied back inside each timed step.  `--impl reference` times the fp64 CPU
oracle on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "mamba130m_layer"
METRIC = "selective-scan fwd B*L*D*N elems/s"
UNIT = "elem/s"
SM_COUNT_B200 = 148
MUFU_EX2_PER_CLK_PER_SM = 16   # SFU ex2 throughput per SM per clock
FALLBACK_HBM_GBS = 6650.0


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return {"hbm_gbs": FALLBACK_HBM_GBS, "sm_max_mhz": 1965.0}, "fallback"


def kernel_source_matches(tag):
    """tag = "<file>@<sha1 prefix>": the kernel source a DRAM-traffic capture
    was taken with; True while csrc/<file> still has that hash."""
    import hashlib
    name, _, digest = tag.partition("@")
    path = os.path.join(ROOT, "selective_state_space_50_b200", "csrc", name)
    if not digest or not os.path.exists(path):
        return False
    with open(path, "rb") as f:
        return hashlib.sha1(f.read()).hexdigest().startswith(digest)


def algorithmic_bytes(w, io_bytes, with_last_state=True, backward=False):
    """HBM bytes a fused forward must move (and, with backward, the backward
    too): every input read once, every output written once."""
    e = w.batch * w.dim * w.seqlen
    bc = w.batch * w.dstate * w.seqlen
    n = e * io_bytes * (3 + 1)                          # u, delta, z in; out
    n += 2 * bc * io_bytes                              # B, C
    n += w.dim * w.dstate * 4 + 2 * w.dim * 4           # A, D, bias
    if with_last_state:
        n += w.batch * w.dim * w.dstate * 4
    if backward:
        # the checkpoints (8 bytes per element each way at N = 16) are this
        # design's choice, not the method's, and are left out
        n += e * io_bytes * 4 + 2 * bc * io_bytes       # u, delta, z, dout, B, C read
        n += e * 4 * 3 + 2 * bc * 4                     # du, ddelta, dz, dB, dC written
        n += w.dim * w.dstate * 4 + 2 * w.dim * 4       # dA, dD, dbias
    return n


# Projections in front of the scan: x_proj (dt_rank + 2 dstate rows) and
# dt_proj (dim rows), bf16; the step is projections + forward scan.
PROJ_WORKLOADS = {"mamba130m_layer_proj": ("mamba130m_layer", 48)}


def projection_bytes(w, dt_rank):
    """HBM bytes of the two projections: x read, the weights, dt_low/B/C
    written, dt_low read again, delta written (bf16)."""
    M1 = dt_rank + 2 * w.dstate
    return 2 * (w.batch * w.dim * w.seqlen + M1 * w.dim + w.batch * M1 * w.seqlen
                + w.dim * dt_rank + w.batch * dt_rank * w.seqlen + w.batch * w.dim * w.seqlen)


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.01):
        self.index, self.period = index, period_s
        self.samples, self.reasons = [], 0
        self._stop = threading.Event()
        self._th = None
        self.max_mhz = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None
            return self

        def run():
            while not self._stop.is_set():
                try:
                    self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
                    self.reasons |= self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                except Exception:
                    pass
                time.sleep(self.period)
        self._th = threading.Thread(target=run, daemon=True)
        self._th.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._th:
            self._th.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        names = [v for k, v in self.REASONS.items() if self.reasons & k and v != "gpu_idle"]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64,
                     device="cuda" if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(seed: int, rank: int) -> int:
    """Seed of a rank's own batch: every rank draws different inputs of the same
    shape (weak scaling, no shared data)."""
    return seed + 7919 * rank


def aggregate_rate(world: int, steps: int, units_per_step: int, t_dev_s: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest
    rank's device time (max over ranks)."""
    return world * steps * units_per_step / max_over_ranks(t_dev_s, world)


def cpu_oracle_rate(w, inp, budget_s: float, nthreads: int = 0, zoh: bool = False):
    """Times the fp64 oracle on whole-batch channel slices until about
    `budget_s` seconds of wall time are spent.  Returns (elem/s, threads, desc)."""
    import oracle
    nthreads = nthreads or oracle.max_threads()
    # slices of 16 channels, all batch rows, full sequence
    step = 16
    done_elems, t_total, slices = 0, 0.0, 0
    d0 = 0
    while t_total < budget_s:
        sl = slice(d0, d0 + step)
        sub = {k: (v[:, sl] if k.split("_f64")[0] in ("u", "delta", "z") else
                   v[sl] if k.split("_f64")[0] in ("A", "D", "delta_bias") else v)
               for k, v in inp.items() if k.endswith("_f64")}
        sub = {k: np.ascontiguousarray(v) for k, v in sub.items()}
        t = time.perf_counter()
        oracle.fwd(sub["u_f64"], sub["delta_f64"], sub["A_f64"], sub["B_f64"], sub["C_f64"],
                   sub["D_f64"], sub["z_f64"], sub["delta_bias_f64"], w.softplus,
                   zoh=zoh, nthreads=nthreads)
        t_total += time.perf_counter() - t
        done_elems += w.batch * step * w.seqlen
        slices += 1
        d0 = (d0 + step) % w.dim
    desc = (f"{slices} slices of {step} channels x batch {w.batch} x seqlen {w.seqlen} "
            f"({done_elems * w.dstate / 1e9:.3f} G state-steps) of the {w.name} forward, "
            f"fp64, {t_total:.1f} s")
    return done_elems * w.dstate / t_total, nthreads, desc


def run_reference(args, world, rank):
    """Reference arm: the fp64 oracle on the host cores, bounded samples."""
    if rank != 0:
        return
    from selective_state_space_50_b200.workloads import WORKLOADS, generate
    w = WORKLOADS[WORKLOAD]
    inp = generate(w, channels=slice(0, 64))
    wsub = w.replace(dim=64)
    import oracle
    nth = oracle.max_threads()
    per_step = slice(0, 8)   # one step = 8 channels x all batch rows x full sequence
    f64 = {k: v for k, v in inp.items() if k.endswith("_f64")}

    def step():
        sub = {}
        for k, v in f64.items():
            base = k[:-4]
            if base in ("u", "delta", "z"):
                sub[k] = np.ascontiguousarray(v[:, per_step])
            elif base in ("A", "D", "delta_bias"):
                sub[k] = np.ascontiguousarray(v[per_step])
            else:
                sub[k] = v
        oracle.fwd(sub["u_f64"], sub["delta_f64"], sub["A_f64"], sub["B_f64"], sub["C_f64"],
                   sub["D_f64"], sub["z_f64"], sub["delta_bias_f64"], True, nthreads=nth)
    for _ in range(args.warmup):
        step()
    t = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t
    elems = args.steps * w.batch * 8 * w.seqlen * w.dstate
    v = elems / dt
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": w.name, "batch": w.batch, "seqlen": w.seqlen, "dim": w.dim,
                       "dstate": w.dstate, "io_dtype": w.io_dtype,
                       "sample": "8 channels x 8 batch rows x 2048 steps per step"},
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": nth, "kind": "oracle",
                             "sample": f"{args.steps} steps of 8 channels x batch {w.batch} x "
                                       f"seqlen {w.seqlen} of the {w.name} forward"},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args, world, rank, local):
    import torch
    from selective_state_space_50_b200 import ssm_scan
    from selective_state_space_50_b200 import dp
    from selective_state_space_50_b200.workloads import WORKLOADS, generate, to_torch

    proj = args.workload in PROJ_WORKLOADS
    if proj:
        base, dt_rank = PROJ_WORKLOADS[args.workload]
        w = WORKLOADS[base].replace(name=args.workload)
    else:
        w = WORKLOADS[args.workload]
    if args.seqlen:   # shorter sequence of the same workload (profiling small cases)
        w = w.replace(seqlen=args.seqlen, name=f"{w.name}_L{args.seqlen}")
    dev = torch.device("cuda", local)
    # every rank processes its own batch of the same shape (weak scaling)
    w_rank = w.replace(seed=rank_seed(w.seed, rank))
    fwdbwd = w.name.startswith("mamba130m_layer_fwdbwd")
    inp = generate(w_rank, with_dout=fwdbwd)
    dv = to_torch(inp, w_rank, dev)
    shape = ssm_scan.make_shape(w.batch, w.dim, w.seqlen, w.dstate, dv["u"].dtype)
    if proj:
        # u is the projections' input x; delta, B and C come from the projections
        from selective_state_space_50_b200.workloads import generate_projection
        pinp = generate_projection(w.batch, w.dim, w.seqlen, w.dstate, dt_rank, w_rank.seed)
        for k in ("x", "W_x", "W_dt"):
            dv[k] = torch.from_numpy(pinp[k].view(np.int16)).view(torch.bfloat16).to(dev)
        dv["u"] = dv["x"]
        bf = dict(device=dev, dtype=torch.bfloat16)
        dv["delta"] = torch.empty(w.batch, w.dim, w.seqlen, **bf)
        dv["B"] = torch.empty(w.batch, w.dstate, w.seqlen, **bf)
        dv["C"] = torch.empty(w.batch, w.dstate, w.seqlen, **bf)
        dt_low = torch.empty(w.batch, dt_rank, w.seqlen, **bf)
    out = torch.empty_like(dv["u"])
    last = torch.empty(w.batch, w.dim, w.dstate, device=dev, dtype=torch.float32)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    nws = 0   # workspace of the two-level scan (forward workloads only)
    if fwdbwd:
        ck = torch.empty(ssm_scan.ckpt_numel(shape), device=dev, dtype=torch.float32)
        f32 = dict(device=dev, dtype=torch.float32)
        grads = {k: torch.empty(dv[src].shape, **f32) for k, src in
                 (("du", "u"), ("ddelta", "u"), ("dz", "u"), ("dA", "A"), ("dB", "B"), ("dC", "C"),
                  ("dD", "D"), ("ddelta_bias", "delta_bias"))}

        def fwd(mid=None):
            # one training step of the scan: forward keeping checkpoints, backward
            # (`mid`, an event recorded between the two launches, times the backward)
            ssm_scan.fwd_raw(shape, dv["u"], dv["delta"], dv["A"], dv["B"], dv["C"], dv["D"],
                             dv["z"], dv["delta_bias"], True, out, last, ck, stream, zoh=args.zoh)
            if mid is not None:
                mid.record(stream)
            ssm_scan.bwd_raw(shape, dv["u"], dv["delta"], dv["A"], dv["B"], dv["C"], dv["D"],
                             dv["z"], dv["delta_bias"], True, dv["dout"], ck, grads["du"],
                             grads["ddelta"], grads["dA"], grads["dB"], grads["dC"], grads["dD"],
                             grads["dz"], grads["ddelta_bias"], None, stream, zoh=args.zoh)
            if world > 1:
                # data parallel: the ranks hold batch rows of one layer, so the
                # parameter gradients are summed over ranks (NCCL all-reduce)
                dp.allreduce_param_grads(grads)
    elif args.segments > 1:
        # the sequence cut into S segments, run with the sharded protocol on
        # this one GPU (pass 1 over all segments, combine, pass 2 over 1..S-1)
        from selective_state_space_50_b200 import seqpar
        S = args.segments
        if w.seqlen % S:
            raise SystemExit("--segments must divide seqlen")
        Ls = w.seqlen // S
        seg_shape = ssm_scan.make_shape(w.batch, w.dim, Ls, w.dstate, dv["u"].dtype)
        pieces = [{k: dv[k][..., s_ * Ls:(s_ + 1) * Ls].contiguous() for k in ("u", "delta", "z", "B", "C")}
                  for s_ in range(S)]
        f32 = dict(device=dev, dtype=torch.float32)
        seg_out = [torch.empty_like(pc["u"]) for pc in pieces]
        seg_last = torch.empty(S, w.batch, w.dim, w.dstate, **f32)
        seg_dsum = torch.empty(S, w.batch, w.dim, **f32)
        h_in = torch.empty(S, w.batch, w.dim, w.dstate, **f32)
        mid = S // 2
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
        seg_times = []

        def run_segment(s_, h0, timed=False):
            pc = pieces[s_]
            ssm_scan.fwd_segment_raw(seg_shape, pc["u"], pc["delta"], dv["A"], pc["B"], pc["C"], dv["D"],
                                     pc["z"], dv["delta_bias"], True, h0, seg_out[s_], seg_last[s_],
                                     None, seg_dsum[s_] if h0 is None else None, stream)
            return seg_out[s_], seg_last[s_], seg_dsum[s_]

        def fwd(record=False):
            for s_ in range(S):
                if record and s_ == mid:
                    ev[0].record(stream)
                run_segment(s_, None)
                if record and s_ == mid:
                    ev[1].record(stream)
            if record:
                ev[2].record(stream)
            ssm_scan.combine_carries_raw(S, w.batch, w.dim, w.dstate, dv["A"], seg_dsum, seg_last, None,
                                         h_in, stream)
            if record:
                ev[3].record(stream)
            for s_ in range(1, S):
                if record and s_ == mid:
                    ev[4].record(stream)
                run_segment(s_, h_in[s_])
                if record and s_ == mid:
                    ev[5].record(stream)
    elif proj:
        def run_proj():
            ssm_scan.projections_raw(shape, dt_rank, dv["x"], dv["W_x"], dv["W_dt"], dt_low,
                                     dv["delta"], dv["B"], dv["C"], stream)

        def fwd():
            run_proj()
            ssm_scan.fwd_raw(shape, dv["u"], dv["delta"], dv["A"], dv["B"], dv["C"], dv["D"],
                             dv["z"], dv["delta_bias"], True, out, last, None, stream)
    else:
        # shapes with long sequences over few channel rows take the two-level
        # scan along the sequence (three launches), with its workspace
        nws = ssm_scan.fwd_workspace_bytes(shape, True, args.zoh)
        ws = torch.empty(nws // 4, device=dev, dtype=torch.float32) if nws else None

        def fwd():
            ssm_scan.fwd_raw(shape, dv["u"], dv["delta"], dv["A"], dv["B"], dv["C"], dv["D"],
                             dv["z"], dv["delta_bias"], True, out, last, None, stream, zoh=args.zoh,
                             workspace=ws)

    for _ in range(max(3, args.warmup)):
        flush.zero_()
        fwd()
    torch.cuda.synchronize()

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    mids = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)] if fwdbwd else None
    with ClockSampler(local) as clk:
        barrier(world)
        torch.cuda.synchronize()
        for i in range(args.steps):
            flush.zero_()
            starts[i].record(stream)
            if fwdbwd:
                fwd(mids[i])
            else:
                fwd()
            ends[i].record(stream)
        torch.cuda.synchronize()
        barrier(world)
    ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    # forward and backward launches of the training step, each on its own
    kern_ms = None
    if fwdbwd:
        kern_ms = {"fwd": sum(s.elapsed_time(m) for s, m in zip(starts, mids)) / args.steps,
                   "bwd": sum(m.elapsed_time(e) for m, e in zip(mids, ends)) / args.steps}
    t_dev = sum(ms) / 1e3
    t_max = max_over_ranks(t_dev, world)
    elems_all = world * args.steps * w.batch * w.dim * w.seqlen * w.dstate
    seg_info = None
    if args.segments > 1:   # one segment's critical path: its pass 1, the combine, its pass 2
        parts = []
        for _ in range(max(3, min(args.steps, 20))):
            flush.zero_()
            fwd(record=True)
            torch.cuda.synchronize()
            parts.append((ev[0].elapsed_time(ev[1]), ev[2].elapsed_time(ev[3]), ev[4].elapsed_time(ev[5])))
        p1, cb, p2 = (statistics.median(x[i] for x in parts) for i in range(3))
        seg_info = {"n": args.segments, "seqlen_per_segment": w.seqlen // args.segments,
                    "pass1_ms": p1, "combine_ms": cb, "pass2_ms": p2, "per_rank_ms": p1 + cb + p2,
                    "exchange_bytes_per_rank": w.batch * w.dim * (w.dstate + 1) * 4,
                    "note": "segments run in turn on one GPU; per_rank_ms is one segment's critical "
                            "path (pass 1 + combine + pass 2, each timed with CUDA events on this GPU); "
                            "the all-gather of the summaries between ranks is not included"}
    t_proj = None
    if proj:   # the two projection launches alone, same L2 flush between steps
        p_s = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        p_e = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        for i in range(args.steps):
            flush.zero_()
            p_s[i].record(stream)
            run_proj()
            p_e[i].record(stream)
        torch.cuda.synchronize()
        t_proj = sum(a.elapsed_time(b) for a, b in zip(p_s, p_e)) / 1e3 / args.steps

    # ---- end to end through the binding, host buffers, copies inside the step
    e2e_steps = max(5, min(args.steps, 50))
    step_inputs = (("x", "W_x", "W_dt", "z", "A", "D", "delta_bias") if proj else
                   ("u", "delta", "z", "B", "C", "A", "D", "delta_bias") + (("dout",) if fwdbwd else ()))
    host = {k: dv[k].cpu().pin_memory() for k in step_inputs}
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    du_h = torch.empty(out.shape, dtype=torch.float32).pin_memory() if fwdbwd else None
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_h.numel() * out_h.element_size() + (du_h.numel() * 4 if fwdbwd else 0)
    e_s = [torch.cuda.Event(enable_timing=True) for _ in range(e2e_steps)]
    e_e = [torch.cuda.Event(enable_timing=True) for _ in range(e2e_steps)]
    dtmp = {k: torch.empty_like(v) for k, v in dv.items() if v is not None}

    # The plain forward pipelines its copies per batch row: row b's inputs go
    # up on one stream while row b - 1 is scanned and row b - 2's output comes
    # back on a third, each row through the public binding.  PCIe carries the
    # copies both ways at once, so the step costs about the inputs' upload.
    pipelined = not (fwdbwd or proj or args.segments > 1) and w.batch > 1
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def e2e_step_pipelined():
        s_in.wait_stream(stream)
        with torch.cuda.stream(s_in):
            for k in ("A", "D", "delta_bias"):
                dtmp[k].copy_(host[k], non_blocking=True)
        for b in range(w.batch):
            with torch.cuda.stream(s_in):
                for k in ("u", "delta", "z", "B", "C"):
                    dtmp[k][b].copy_(host[k][b], non_blocking=True)
                ev_in = torch.cuda.Event()
                ev_in.record(s_in)
            stream.wait_event(ev_in)
            sl = slice(b, b + 1)
            ssm_scan.selective_scan_fwd(dtmp["u"][sl], dtmp["delta"][sl], dtmp["A"], dtmp["B"][sl],
                                        dtmp["C"][sl], dtmp["D"], dtmp["z"][sl], dtmp["delta_bias"],
                                        True, return_last_state=True, out=out[sl], zoh=args.zoh,
                                        stream=stream)
            ev_c = torch.cuda.Event()
            ev_c.record(stream)
            s_out.wait_event(ev_c)
            with torch.cuda.stream(s_out):
                out_h[b].copy_(out[b], non_blocking=True)
        stream.wait_stream(s_out)

    def e2e_step():
        if pipelined:
            e2e_step_pipelined()
            return
        for k, t in host.items():
            dtmp[k].copy_(t, non_blocking=True)
        if args.segments > 1:
            o, _ = seqpar.cuda_forward_segments(dtmp["u"], dtmp["delta"], dtmp["A"], dtmp["B"], dtmp["C"],
                                                dtmp["D"], dtmp["z"], dtmp["delta_bias"], True,
                                                nseg=args.segments)
            out_h.copy_(o, non_blocking=True)
            return
        if proj:
            d_, B_, C_, _ = ssm_scan.selection_projections(dtmp["x"], dtmp["W_x"], dtmp["W_dt"], w.dstate)
            o, _, _ = ssm_scan.selective_scan_fwd(dtmp["x"], d_, dtmp["A"], B_, C_, dtmp["D"], dtmp["z"],
                                                  dtmp["delta_bias"], True, return_last_state=True,
                                                  out=out)
            out_h.copy_(o, non_blocking=True)
            return
        o, _, ckp = ssm_scan.selective_scan_fwd(dtmp["u"], dtmp["delta"], dtmp["A"], dtmp["B"],
                                                dtmp["C"], dtmp["D"], dtmp["z"], dtmp["delta_bias"],
                                                True, return_last_state=True, out=out,
                                                return_ckpt=fwdbwd, zoh=args.zoh)
        if fwdbwd:
            g = ssm_scan.selective_scan_bwd(dtmp["u"], dtmp["delta"], dtmp["A"], dtmp["B"],
                                            dtmp["C"], dtmp["D"], dtmp["z"], dtmp["delta_bias"],
                                            True, dtmp["dout"], ckpt=ckp, zoh=args.zoh)
            du_h.copy_(g["du"], non_blocking=True)
        out_h.copy_(o, non_blocking=True)
    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    for i in range(e2e_steps):
        flush.zero_()
        e_s[i].record(stream)
        e2e_step()
        e_e[i].record(stream)
    torch.cuda.synchronize()
    t_e2e = max_over_ranks(sum(s.elapsed_time(e) for s, e in zip(e_s, e_e)) / 1e3, world)
    e2e_val = world * e2e_steps * w.batch * w.dim * w.seqlen * w.dstate / t_e2e

    if rank != 0:
        return
    chunked = not (fwdbwd or proj or args.segments > 1) and nws > 0
    peaks, peak_src = measured_peaks()
    mean_s = t_dev / args.steps
    # The roofline is the dominant kernel's: the forward scan, or in the
    # training step the backward (timed on its own between events).  Each
    # needs one exponential per (step, state): Ā of the recurrence, and in the
    # backward Ā of the reverse sweep (its minimum with checkpoints).
    ex2 = w.batch * w.dim * w.seqlen * w.dstate
    kern_s = kern_ms["bwd"] / 1e3 if fwdbwd else mean_s
    sm_max = float(peaks.get("sm_max_mhz") or 1965.0)
    mufu_peak = SM_COUNT_B200 * MUFU_EX2_PER_CLK_PER_SM * sm_max * 1e6
    achieved = ex2 / kern_s
    alg_bytes = algorithmic_bytes(w, 2 if w.io_dtype == "bf16" else 4, backward=fwdbwd)
    # bytes of the dominant kernel alone (the backward's reads and writes)
    k_bytes = (alg_bytes - algorithmic_bytes(w, 2 if w.io_dtype == "bf16" else 4)
               if fwdbwd else alg_bytes)
    # DRAM bytes of one launch of the dominant kernel, from the ncu capture
    # named beside it (profiles/dram_traffic.txt); None where there is none
    traffic, traffic_src = None, None
    tp = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    key = ("ssm_bwd_" if fwdbwd else "ssm_fwd_") + w.name
    if os.path.exists(tp) and not proj and not chunked and not args.zoh:
        with open(tp) as f:
            for line in f:
                parts = line.split()
                if len(parts) >= 2 and not line.startswith("#") and parts[0] == key:
                    traffic = int(parts[1])
                    traffic_src = "profiles/" + parts[2] if len(parts) > 2 else "profiles/dram_traffic.txt"
                    if len(parts) > 3 and not kernel_source_matches(parts[3]):
                        traffic = None
                        traffic_src += " (stale: " + parts[3].split("@")[0] + " changed since the capture)"
    line = {
        "metric": METRIC, "value": elems_all / t_max, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": max(3, args.warmup),
        "ms_per_step": t_max / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "seqlen": w.seqlen, "dim": w.dim,
                   "dstate": w.dstate, "io_dtype": w.io_dtype, "state_dtype": "f32",
                   "parallelism": (f"data parallel x{world} (own batch rows per rank; parameter "
                                   f"gradients all-reduced)" if fwdbwd and world > 1 else
                                   f"replicas x{world} (independent batches)"),
                   "l2": "flushed between steps (256 MiB write, outside the timed events)"},
        "gbs": alg_bytes / mean_s / 1e9,
        "roofline": {"bound": "alu", "kernel": "backward" if fwdbwd else "forward",
                     "achieved": achieved / 1e12, "peak": mufu_peak / 1e12,
                     "unit": "Tex2/s", "frac": achieved / mufu_peak, "traffic": traffic,
                     "traffic_source": traffic_src,
                     "peak_source": f"148 SMs x 16 ex2/clk x {sm_max:.0f} MHz (SFU)",
                     "hbm": {"achieved_gbs": k_bytes / kern_s / 1e9,
                             "peak_gbs": float(peaks["hbm_gbs"]),
                             "frac": k_bytes / kern_s / 1e9 / float(peaks["hbm_gbs"]),
                             "peak_source": peak_src, "alg_bytes": k_bytes}},
        "clocks": clk.summary(),
        "e2e": {"value": e2e_val, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "pipeline": ("per batch row: upload, scan and download on three streams"
                             if pipelined else "one upload, the step, one download")},
        # segments: S pass-1 scans (the TMA forward also sums Δ), the combine,
        # S - 1 pass-2 scans
        "gpu_launches": args.steps * (3 if proj else 2 if fwdbwd else
                                      (2 * args.segments if args.segments > 1 else
                                       3 if chunked else 1)),
    }
    if kern_ms:
        line["kernels_ms"] = dict(kern_ms, note=(
            "CUDA events on the launching stream around the forward launch and around the "
            "backward call (its gradient zero-fills included"
            + (", and the parameter-gradient all-reduce" if world > 1 else "") + ")"))
    if args.zoh:
        line["config"]["discretization"] = "zero-order hold"
    if chunked:
        line["config"]["step"] = ("two-level scan along the sequence: chunk summaries, carry "
                                  "combine, every chunk from its carry-in (3 launches)")
    if seg_info:
        line["segments"] = seg_info
        line["config"]["step"] = (f"sequence cut into {args.segments} segments: pass 1 over all, "
                                  f"carry combine, pass 2 over segments 1..{args.segments - 1}")
    if proj:
        pb = projection_bytes(w, dt_rank)
        flops = 2 * w.batch * w.seqlen * w.dim * (2 * dt_rank + 2 * w.dstate)
        line["config"]["dt_rank"] = dt_rank
        line["config"]["step"] = "x_proj + dt_proj (tcgen05) + forward scan"
        line["projections"] = {"ms": t_proj * 1e3, "alg_bytes": pb, "flops": flops,
                               "hbm": {"achieved_gbs": pb / t_proj / 1e9,
                                       "peak_gbs": float(peaks["hbm_gbs"]),
                                       "frac": pb / t_proj / 1e9 / float(peaks["hbm_gbs"])},
                               "tflops": flops / t_proj / 1e12}
    if world == 1 and not args.no_cpu_baseline:
        rate, cores, desc = cpu_oracle_rate(w, inp, args.cpu_budget, zoh=args.zoh)
        if proj:
            # the oracle's projections on one batch row x 256 steps (all channels)
            import oracle
            sl = slice(0, min(256, w.seqlen))
            t0 = time.perf_counter()
            oracle.projections(pinp["x_f64"][:1, :, sl], pinp["W_x_f64"], pinp["W_dt_f64"],
                               dt_rank, w.dstate)
            tp_s = time.perf_counter() - t0
            r_proj = w.dim * (sl.stop - sl.start) * w.dstate / tp_s
            rate = 1.0 / (1.0 / rate + 1.0 / r_proj)
            desc += f"; projections: 1 batch row x {sl.stop} steps, fp64, {tp_s:.2f} s"
        line["cpu_baseline"] = {"value": rate, "unit": UNIT, "cores": cores, "kind": "oracle",
                                "sample": desc}
    print(json.dumps(line), flush=True)


def run_decode(args, world, rank, local):
    """One decoding step (ssm_selective_state_update) at the Mamba-2.8B layer
    width: batch 64 sequences, dim 5120, dstate 16, bf16 io, fp32 state kept
    on the device.  Memory-bound: reported against the HBM roofline."""
    import torch
    import oracle
    from selective_state_space_50_b200 import ssm_scan
    from selective_state_space_50_b200.workloads import Workload, generate, to_torch

    w = Workload("decode_step_2p8b", 64, 1, 5120, 16, "bf16", seed=rank_seed(1005, rank),
                 D_dist="u0.5_1.5")
    dev = torch.device("cuda", local)
    inp = generate(w)
    dv = to_torch(inp, w, dev)
    sq = {k: (dv[k][..., 0].contiguous() if dv[k] is not None and k in ("u", "delta", "z", "B", "C")
              else dv[k]) for k in dv}
    st0 = np.random.default_rng(w.seed).standard_normal((w.batch, w.dim, w.dstate)).astype(np.float32)
    state = torch.from_numpy(st0).to(dev)
    out = torch.empty_like(sq["u"])
    shape = ssm_scan.make_shape(w.batch, w.dim, 1, w.dstate, sq["u"].dtype)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def step():
        ssm_scan.state_update_raw(shape, state, sq["u"], sq["delta"], sq["A"], sq["B"], sq["C"],
                                  sq["D"], sq["z"], sq["delta_bias"], True, out, stream)

    for _ in range(max(3, args.warmup)):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    with ClockSampler(local) as clk:
        barrier(world)
        torch.cuda.synchronize()
        for i in range(args.steps):
            flush.zero_()
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        torch.cuda.synchronize()
        barrier(world)
    t_dev = sum(s.elapsed_time(e) for s, e in zip(starts, ends)) / 1e3
    t_max = max_over_ranks(t_dev, world)
    units = w.batch * w.dim * w.dstate

    # end to end: the token's inputs from pinned host memory, the output back;
    # the state stays on the device (as in a decoding loop)
    host = {k: sq[k].cpu().pin_memory() for k in ("u", "delta", "z", "B", "C")}
    dtmp = {k: torch.empty_like(sq[k]) for k in host}
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_h.numel() * out_h.element_size()
    e2e_steps = max(5, min(args.steps, 50))
    e_s = [torch.cuda.Event(enable_timing=True) for _ in range(e2e_steps)]
    e_e = [torch.cuda.Event(enable_timing=True) for _ in range(e2e_steps)]

    def e2e_step():
        for k, t in host.items():
            dtmp[k].copy_(t, non_blocking=True)
        o = ssm_scan.selective_state_update(state, dtmp["u"], dtmp["delta"], sq["A"], dtmp["B"],
                                            dtmp["C"], sq["D"], dtmp["z"], sq["delta_bias"], True,
                                            out=out)
        out_h.copy_(o, non_blocking=True)
    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    for i in range(e2e_steps):
        flush.zero_()
        e_s[i].record(stream)
        e2e_step()
        e_e[i].record(stream)
    torch.cuda.synchronize()
    t_e2e = max_over_ranks(sum(s.elapsed_time(e) for s, e in zip(e_s, e_e)) / 1e3, world)
    if rank != 0:
        return
    peaks, peak_src = measured_peaks()
    mean_s = t_dev / args.steps
    es_io = 2
    alg = (2 * 4 * units + 4 * es_io * w.batch * w.dim + 2 * es_io * w.dstate * w.batch
           + 4 * w.dim * w.dstate + 8 * w.dim)
    line = {
        "metric": "selective-state-update B*D*N elems/s", "value": world * args.steps * units / t_max,
        "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": max(3, args.warmup),
        "ms_per_step": t_max / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "dim": w.dim, "dstate": w.dstate,
                   "io_dtype": w.io_dtype, "state_dtype": "f32",
                   "parallelism": f"replicas x{world} (independent batches)",
                   "l2": "flushed between steps (256 MiB write, outside the timed events)"},
        "roofline": {"bound": "hbm", "achieved": alg / mean_s / 1e9, "peak": float(peaks["hbm_gbs"]),
                     "unit": "GB/s", "frac": alg / mean_s / 1e9 / float(peaks["hbm_gbs"]),
                     "traffic": None, "peak_source": peak_src, "alg_bytes": alg},
        "clocks": clk.summary(),
        "e2e": {"value": world * e2e_steps * units / t_e2e, "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": args.steps,
    }
    if world == 1 and not args.no_cpu_baseline:
        st64 = st0.astype(np.float64)
        t0 = time.perf_counter()
        n = 0
        while time.perf_counter() - t0 < min(args.cpu_budget, 5.0) or n == 0:
            oracle.step(st64, inp["u_f64"][..., 0], inp["delta_f64"][..., 0], inp["A_f64"],
                        inp["B_f64"][..., 0], inp["C_f64"][..., 0], inp["D_f64"], inp["z_f64"][..., 0],
                        inp["delta_bias_f64"], True)
            n += 1
        el = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": n * units / el, "unit": UNIT, "cores": oracle.max_threads(),
                                "kind": "oracle",
                                "sample": f"{n} full steps of {w.name} (fp64), {el:.1f} s"}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--workload", default=WORKLOAD,
                    help="workload to time (default: the Mamba-130M layer shape)")
    ap.add_argument("--seqlen", type=int, default=0,
                    help="override the workload's sequence length (for profiling small cases)")
    ap.add_argument("--zoh", action="store_true",
                    help="zero-order-hold discretisation (forward workloads)")
    ap.add_argument("--segments", type=int, default=1,
                    help="run the forward as S sequence segments with the sharded protocol")
    ap.add_argument("--decode", action="store_true",
                    help="time the single-step recurrent update instead of the scan")
    args = ap.parse_args()
    if args.zoh and (args.decode or args.segments > 1 or args.workload in PROJ_WORKLOADS):
        ap.error("--zoh applies to the scan workloads (not --decode, --segments or the projections)")
    if args.segments > 1 and (args.decode or args.workload in PROJ_WORKLOADS
                              or args.workload.endswith("fwdbwd")):
        ap.error("--segments applies to the forward scan workloads")
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        elif args.decode:
            run_decode(args, world, rank, local)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
