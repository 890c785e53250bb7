"""Benchmark of the MoE expert-parallel token round trip on B200.

One step = one pass of the whole round trip over one batch: route ->
dispatch -> grouped SwiGLU FFN (gate/up, down) -> combine, through the C ABI.
Default workload: the GPT-OSS-20B-shaped layer with balanced routing
(T=4096, H=2880, I=3072, E=32, top-4, R=8 logical ranks, bf16).

Prints ONE JSON line on rank 0.  Under torchrun each GPU runs its own
independent copy of the layer on its own batch (weak scaling, no data-path
collective); time is the max over ranks.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

METRIC = "MoE-layer tokens/s; dispatch+combine HBM GB/s; grouped-GEMM TFLOP/s vs peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 512 << 20  # > 126 MB of L2
HOLD_CYCLES = 400_000  # GPU spin before each timed step (~0.2 ms), outside the timed events


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_sha() -> str:
    h = hashlib.sha256()
    for name in ("ffn_tc.cuh", "ffn_tc2.cuh", "common.cuh"):
        with open(os.path.join(ROOT, "token_dispatch_combine_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def dram_traffic(workload: str, gather: bool = False):
    """Per-launch DRAM bytes of the gate/up kernel (its gathering form when `gather`)
    from the committed ncu summary, if taken on the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    sha = kernel_source_sha()
    for line in open(path):
        parts = line.split()
        if len(parts) >= 4 and not line.startswith("#") and parts[0] == workload \
                and parts[1] == ("gate_up_gather" if gather else "gate_up") and parts[3] == sha:
            return int(float(parts[2]))
    return None


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML during the timed region."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
        "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
    }

    def __init__(self, device_index: int):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nvml = None
        self.t = threading.Thread(target=self._run, daemon=True)

    def _sample(self):
        n = self.nvml
        self.samples.append(n.nvmlDeviceGetClockInfo(self.h, n.NVML_CLOCK_SM))
        mask = n.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        for name, bit in self.REASONS.items():
            if mask & bit and name != "gpu_idle":
                self.reasons.add(name)

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception:
                return
            time.sleep(0.005)

    def __enter__(self):
        if self.nvml:
            self.t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.nvml:
            self.t.join()
            try:
                self._sample()
            except Exception:
                pass

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["nvml unavailable"]}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(values, world):
    """Element-wise max of per-rank timings (the slowest rank sets the job's time)."""
    import torch
    if world == 1:
        return list(values)
    import torch.distributed as dist
    device = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def algorithmic(wl):
    b = 2 if wl.dtype == "bf16" else 4
    S = wl.S
    return {
        "dispatch_bytes": wl.T * wl.H * b + S * wl.H * b + 12 * S,  # x read, x_disp write, ids/ranks/maps
        "combine_bytes": S * wl.H * b + wl.T * wl.H * b + 8 * S,  # y_disp read, y write, w + slot_to_row
        "route_bytes": wl.T * wl.E * 4 + wl.T * wl.k * 8,
        "router_bytes": wl.T * wl.H * 2 + wl.E * wl.H * 2 + wl.T * wl.k * 8,  # x, W_r read; ids, w written
        "gateup_flops": 4.0 * S * wl.H * wl.I,
        "down_flops": 2.0 * S * wl.H * wl.I,
    }


def gemm_bounds(wl, counts, gather, peaks):
    """Roofline of the two grouped GEMMs from the layer's expert counts.

    Per projection: algorithmic FLOPs and bytes (weights of the experts that have rows, the A rows
    read once -- x itself when the gate/up projection gathers, the k-fold re-reads being L2 hits --
    and the output written once), which of the two bounds the launch (time at the measured peak),
    and the per-expert bound sum_e max(F_e / P_F, B_e / P_B) (each expert's weights stream while its
    rows' products run)."""
    b = 2 if wl.dtype == "bf16" else 4
    H, I, S, T = wl.H, wl.I, wl.S, wl.T
    P_F, P_B = peaks["bf16_tflops"] * 1e12, peaks["hbm_gbs"] * 1e9
    counts = np.asarray(counts, np.float64)
    active = counts > 0
    out = {}
    for proj, (w_elems, n_out, k_in, fl_per_row) in {
            "gate_up": (2 * H * I, I, H, 4.0 * H * I), "down": (I * H, H, I, 2.0 * H * I)}.items():
        flops = fl_per_row * S
        a_rows = (T if (gather and proj == "gate_up") else S) * k_in * b
        nbytes = active.sum() * w_elems * b + a_rows + S * n_out * b
        f_e = fl_per_row * counts
        b_e = active * w_elems * b + counts * (k_in + n_out) * b
        out[proj] = {"flops": flops, "bytes": float(nbytes), "t_tensor": flops / P_F, "t_hbm": nbytes / P_B,
                     "t_per_expert": float(np.maximum(f_e / P_F, b_e / P_B).sum())}
    return out


# --------------------------------------------------------------------------- CPU oracle legs
def oracle_sample_step(wl, x, logits, wg, wu, wd, n_tok, rng):
    """The oracle's round trip on a batch of n_tok tokens of the workload."""
    import oracle
    idx = np.sort(rng.choice(wl.T, size=n_tok, replace=False))
    t0 = time.perf_counter()
    oracle.round_trip(x[idx], logits[idx], wl.k, wl.E, wl.R, wg, wu, wd)
    return time.perf_counter() - t0


def size_oracle_sample(wl, x, logits, wg, wu, wd, target_s, rng):
    n = max(1, min(wl.T, 4))
    dt = oracle_sample_step(wl, x, logits, wg, wu, wd, n, rng)
    per_tok = dt / n
    return int(max(1, min(wl.T, target_s / max(per_tok, 1e-9)))), per_tok


def cpu_cores():
    n = os.environ.get("OMP_NUM_THREADS")
    return int(n) if n else (os.cpu_count() or 1)


def host_inputs(wl):
    x = wl.x()
    logits = wl.logits(synth.bf16_bits_to_f32(x) if wl.dtype == "bf16" else x)
    return x, logits, wl.w_gate(), wl.w_up(), wl.w_down()


def run_reference(args, wl):
    """Reference arm: the CPU oracle, timed on the host cores, rank 0 only."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    x, logits, wg, wu, wd = host_inputs(wl)
    rng = np.random.default_rng(0)
    n_tok, _ = size_oracle_sample(wl, x, logits, wg, wu, wd, target_s=2.0, rng=rng)
    for _ in range(args.warmup):
        oracle_sample_step(wl, x, logits, wg, wu, wd, n_tok, rng)
    times = [oracle_sample_step(wl, x, logits, wg, wu, wd, n_tok, rng) for _ in range(args.steps)]
    total = sum(times)
    value = n_tok * args.steps / total
    sample = f"{n_tok} of {wl.T} tokens per step (whole round trip on that batch, same layer)"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(wl),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cpu_cores(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_dict(wl):
    return {"workload": wl.name, "T": wl.T, "H": wl.H, "I": wl.I, "E": wl.E, "k": wl.k, "R": wl.R,
            "dtype": wl.dtype, "routing_bias": wl.bias, "seed": wl.seed,
            "l2": f"flushed between steps ({L2_FLUSH_BYTES >> 20} MiB write, then read back)"}


# --------------------------------------------------------------------------- our arm
def run_ours(args, wl):
    import torch

    from token_dispatch_combine_b200 import (FFN_DOWN, FFN_GATE_UP, FFN_TILING_PAIR, MoERoundTrip, moe_ffn_tiling_for,
                                             moe_get_error, moe_set_ffn_tiling)
    moe_set_ffn_tiling({"auto": 0, "single": 1, "pair": 2}[args.ffn_tiling])
    world, rank, local = dist_setup(args)
    dev = torch.device("cuda", torch.cuda.current_device())
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32

    x_np, logits_np, wg_np, wu_np, wd_np = host_inputs(wl)

    def up(a):
        t = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a)
        return t.to(dev).view(dt) if a.dtype == np.uint16 else t.to(dev)

    x, logits = up(x_np), up(logits_np)
    wg, wu, wd = up(wg_np), up(wu_np), up(wd_np)
    rc = args.route_counts == "on"
    rt = MoERoundTrip(wl.T, wl.H, wl.I, wl.E, wl.k, wl.R, dt, device=dev,
                      gather={"auto": "auto", "rows": False, "gather": True}[args.dispatch], route_counts=rc,
                      combine_in_down=args.combine_in_down == "on")
    gather = rt.gather
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
    flush_max = torch.empty((), dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()

    def step(ev):
        ev[0].record(stream)
        rt.route(logits)
        ev[1].record(stream)
        rt.dispatch(x)
        ev[2].record(stream)
        rt.gate_up(wg, wu)
        ev[3].record(stream)
        rt.down(wd)
        ev[4].record(stream)
        rt.combine()
        ev[5].record(stream)

    def flush_and_hold():
        # Outside the timed events: evict L2 by writing a buffer 4x its size, then
        # read that buffer back so L2 holds clean lines of it (a write alone leaves
        # ~126 MB of dirty lines that the timed step would have to write back);
        # then keep the GPU busy for ~0.2 ms so the host has enqueued the whole
        # step before the GPU reaches it (the stage events then measure GPU time,
        # not Python call overhead).
        flush.zero_()
        torch.amax(flush, dim=0, out=flush_max)
        torch.cuda._sleep(HOLD_CYCLES)

    for _ in range(args.warmup):
        flush_and_hold()
        step([torch.cuda.Event(enable_timing=True) for _ in range(6)])
    st, bits = moe_get_error()
    if st != 0:
        raise RuntimeError(f"device error word {bits} during warm-up")
    expert_counts = rt.disp.expert_counts.cpu().numpy()  # outside the timed region

    # Timed region: K whole steps, one event pair per step (no events between stages).
    def whole_step(a, b):
        a.record(stream)
        rt.route(logits)
        rt.dispatch(x)
        rt.gate_up(wg, wu)
        rt.down(wd)
        rt.combine()
        b.record(stream)

    pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        for a, b in pairs:
            flush_and_hold()  # inputs start cold in L2
            whole_step(a, b)
        torch.cuda.synchronize()
    barrier(world)
    step_ms = sum(a.elapsed_time(b) for a, b in pairs) / args.steps

    # Instrumented pass (same work, events between the five stages) for the per-stage breakdown.
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    for i in range(args.steps):
        flush_and_hold()
        step(events[i])
    torch.cuda.synchronize()
    stage = np.zeros(5)
    for ev in events:
        stage += [ev[j].elapsed_time(ev[j + 1]) for j in range(5)]
    stage /= args.steps  # ms per step per stage: route, dispatch, gate_up, down, combine

    # The dispatch+combine metric is about the row-moving dispatch: when the step gathers its
    # rows in the gate/up projection, measure dispatch (with rows) and combine on a second,
    # row-moving round trip of the same layer.
    if gather or rt.combine_in_down:  # (the metric's combine is moe_combine on y_disp)
        rt_dc = MoERoundTrip(wl.T, wl.H, wl.I, wl.E, wl.k, wl.R, dt, device=dev, gather=False, route_counts=rc)
        rt_dc.forward(x, logits, wg, wu, wd)
        dc_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
        for ev in dc_ev:
            flush_and_hold()
            ev[0].record(stream)
            rt_dc.dispatch(x)
            ev[1].record(stream)
            flush_and_hold()
            ev[2].record(stream)
            rt_dc.combine()
            ev[3].record(stream)
        torch.cuda.synchronize()
        dc_stage = [sum(ev[0].elapsed_time(ev[1]) for ev in dc_ev) / args.steps,
                    sum(ev[2].elapsed_time(ev[3]) for ev in dc_ev) / args.steps]
    else:
        rt_dc = rt
        dc_stage = [float(stage[1]), float(stage[4])]

    # Dispatch and combine back to back (same bytes: combine reads the previous step's y_disp),
    # one event pair around both, L2 flushed before: their cost without the per-stage events.
    pair = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for a, b in pair:
        flush_and_hold()
        a.record(stream)
        rt_dc.dispatch(x)
        rt_dc.combine()
        b.record(stream)
    torch.cuda.synchronize()
    dc_pair_ms = sum(a.elapsed_time(b) for a, b in pair) / args.steps
    # Dispatch + combine as a stream of layers: 4 independent buffer sets (x, dispatched rows,
    # y_disp, y: ~1.3 GB, far beyond the 126 MB L2) visited in turn, 20 pairs under one event pair.
    # Launch latency is then overlapped as it is inside a step, and no pair finds its data in L2.
    sets = [MoERoundTrip(wl.T, wl.H, wl.I, wl.E, wl.k, wl.R, dt, device=dev, gather=False, route_counts=rc)
            for _ in range(4)]
    xs = [x.clone() for _ in sets]
    for r_, x_ in zip(sets, xs):
        r_.route(logits)
        r_.dispatch(x_)
        r_.y_disp.copy_(rt_dc.y_disp)
    n_pairs = 20
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    flush_and_hold()
    a.record(stream)
    for i in range(n_pairs):
        sets[i % 4].dispatch(xs[i % 4])
        sets[i % 4].combine()
    b.record(stream)
    torch.cuda.synchronize()
    dc_stream_ms = a.elapsed_time(b) / n_pairs
    del sets, xs
    if rt_dc is not rt:
        del rt_dc

    # The masking form's return path (moe_combine_rank_partials + moe_reduce_rank_partials) in
    # place of combine, on this step's y_disp: R per-rank partial planes, then their rank-ordered
    # sum; L2 flushed before each kernel.
    masked = None
    if wl.R > 1:
        from token_dispatch_combine_b200 import moe_combine_rank_partials, moe_reduce_rank_partials
        y_part = torch.empty((wl.R, wl.T, wl.H), dtype=dt, device=dev)
        y_m = torch.empty((wl.T, wl.H), dtype=dt, device=dev)
        mev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
        for ev in mev:
            flush_and_hold()
            ev[0].record(stream)
            moe_combine_rank_partials(rt.y_disp, rt.topk_w, rt.topk_ids, rt.disp.slot_to_row, wl.E, wl.R, y_part)
            ev[1].record(stream)
            flush_and_hold()
            ev[2].record(stream)
            moe_reduce_rank_partials(y_part, y_m)
            ev[3].record(stream)
        torch.cuda.synchronize()
        st, bits = moe_get_error()
        if st != 0:
            raise RuntimeError(f"device error word {bits} in the masking form")
        b_ = 2 if wl.dtype == "bf16" else 4
        part_us = statistics.median(ev[0].elapsed_time(ev[1]) for ev in mev) * 1e3
        red_us = statistics.median(ev[2].elapsed_time(ev[3]) for ev in mev) * 1e3
        part_bytes = wl.S * wl.H * b_ + wl.R * wl.T * wl.H * b_ + 12 * wl.S
        red_bytes = wl.R * wl.T * wl.H * b_ + wl.T * wl.H * b_
        masked = {"rank_partials_us": part_us, "reduce_us": red_us,
                  "rank_partials_gbs": part_bytes / (part_us * 1e-6) / 1e9,
                  "reduce_gbs": red_bytes / (red_us * 1e-6) / 1e9,
                  "extra_us_vs_combine": part_us + red_us - float(stage[4]) * 1e3,
                  "bytes": "partials S*H*b + R*T*H*b + 12*S; reduction R*T*H*b + T*H*b",
                  "timing": "events per kernel, L2 flushed before each, median of the steps"}
        del y_part, y_m

    # The exchange between ranks (moe_ep_*), its R ranks emulated on this GPU with their own
    # buffers (the step of ep_round_trip_one_gpu, phase by phase): every rank's plan, the counts
    # exchange (a host copy, outside the events), every rank's pack into the others' receive
    # buffers, every rank's local experts over what it received, the partials' return and every
    # rank's sum.  L2 flushed before the plan.  Its pack would cross NVLink on R GPUs.
    ep_info = None
    ep_bytes = wl.R * (wl.T // max(wl.R, 1)) * wl.k * (wl.H + wl.I) * (2 if wl.dtype == "bf16" else 4) * wl.R
    if 1 < wl.R <= 64 and wl.T % wl.R == 0 and ep_bytes < (8 << 30):
        from token_dispatch_combine_b200 import MoEEPRank
        q = wl.T // wl.R
        ranks = [MoEEPRank(r, wl.R, q, wl.H, wl.I, wl.E, wl.k, dt, device=dev, recv_capacity=wl.T)
                 for r in range(wl.R)]
        xs = [x[r * q:(r + 1) * q] for r in range(wl.R)]
        lgs = [logits[r * q:(r + 1) * q].contiguous() for r in range(wl.R)]
        EL = wl.E // wl.R
        wsl = [(wg[d * EL:(d + 1) * EL], wu[d * EL:(d + 1) * EL], wd[d * EL:(d + 1) * EL]) for d in range(wl.R)]
        phases = np.zeros(5)
        n_ep = max(3, min(args.steps, 10))
        for it in range(n_ep + 1):  # the first is a warm-up
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(7)]
            flush_and_hold()
            ev[0].record(stream)
            for r_, lg_ in zip(ranks, lgs):
                r_.route_and_plan(lg_)
            ev[1].record(stream)
            counts = torch.stack([r_.plan.send_counts for r_ in ranks]).cpu().numpy()
            for r_ in ranks:
                r_.set_counts(counts)
            # after that host round trip the GPU would wait for each launch of the host: hold it
            # (~6 ms) while the host enqueues the rest, so the phase events measure GPU time
            torch.cuda._sleep(HOLD_CYCLES * 30)
            ev[2].record(stream)
            for r_, x_ in zip(ranks, xs):
                r_.pack_to(x_, ranks)
            ev[3].record(stream)
            for r_, w_ in zip(ranks, wsl):
                r_.experts(*w_)
            ev[4].record(stream)
            for r_ in ranks:
                r_.return_to(ranks)
            ev[5].record(stream)
            for r_ in ranks:
                r_.finish()
            ev[6].record(stream)
            torch.cuda.synchronize()
            if it:
                phases += [ev[0].elapsed_time(ev[1]), ev[2].elapsed_time(ev[3]), ev[3].elapsed_time(ev[4]),
                           ev[4].elapsed_time(ev[5]), ev[5].elapsed_time(ev[6])]
        phases /= n_ep
        st, bits = moe_get_error()
        if st != 0:
            raise RuntimeError(f"device error word {bits} in the exchange between ranks")
        rows = int(counts.sum())
        b_ = 2 if wl.dtype == "bf16" else 4
        pack_bytes = rows * (2 * wl.H * b_ + 16 * wl.k)
        ep_info = {"ranks": wl.R, "tokens_per_rank": q, "rows_sent": rows, "slots": wl.S,
                   "plan_us": phases[0] * 1e3, "pack_us": phases[1] * 1e3, "experts_us": phases[2] * 1e3,
                   "return_us": phases[3] * 1e3, "finish_us": phases[4] * 1e3,
                   "pack_gbs": pack_bytes / (phases[1] * 1e-3) / 1e9,
                   "timing": "all R ranks on this GPU, events per phase summed over the ranks, L2 flushed "
                             "before the plan; counts exchanged through the host outside the events, then the "
                             "GPU held while the host enqueues the later phases; pack bytes = rows sent x (read "
                             "+ write of a row) + ids/weights"}
        del ranks

    # The router affinities fused with the top-k (moe_router_topk): logits = x W_r^T + bias on
    # tensor cores, then route's selection; L2 flushed before each call.  Not part of the step
    # above, which starts from given logits.
    router_ms = None
    if wl.dtype == "bf16" and wl.E <= 256:
        from token_dispatch_combine_b200 import moe_router_topk
        w_router = torch.from_numpy(np.ascontiguousarray(wl.router_weight().T)).to(dev).to(torch.bfloat16)
        r_bias = torch.from_numpy(wl.router_bias().astype(np.float32)).to(dev) if wl.bias != "none" else None
        r_ids = torch.empty((wl.T, wl.k), dtype=torch.int32, device=dev)
        r_w = torch.empty((wl.T, wl.k), dtype=torch.float32, device=dev)
        for _ in range(3):
            moe_router_topk(x, w_router, wl.k, bias=r_bias, topk_ids=r_ids, topk_w=r_w)
        rev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        for a, b in rev:
            flush_and_hold()
            a.record(stream)
            moe_router_topk(x, w_router, wl.k, bias=r_bias, topk_ids=r_ids, topk_w=r_w)
            b.record(stream)
        torch.cuda.synchronize()
        router_ms = sum(a.elapsed_time(b) for a, b in rev) / args.steps
        del w_router, r_ids, r_w
    # The whole step replayed from a CUDA graph (one launch from the host per step), L2 flushed
    # before each replay outside the graph.
    graph_ms, graph_err = None, None
    try:
        g = rt.capture(x, logits, wg, wu, wd)
        g.replay()
        torch.cuda.synchronize()
        ev_g = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(args.steps)]
        for a, b in ev_g:
            flush_and_hold()
            a.record(stream)
            g.replay()
            b.record(stream)
        torch.cuda.synchronize()
        graph_ms = statistics.median(a.elapsed_time(b) for a, b in ev_g)
        del g
    except Exception as exc:  # reported in the line; the eager numbers stand on their own
        graph_err = f"{type(exc).__name__}: {exc}"[:200]
    st, bits = moe_get_error()
    if st != 0:
        raise RuntimeError(f"device error word {bits} in the graph replay")

    # Expert placement with replicas (one spare physical slot per logical rank), planned on the
    # warm-up's expert counts: the busiest rank's rows before and after, the remap kernel's time,
    # and the whole balanced step (route, remap, dispatch, FFN, combine over the replicas).
    eplb = None
    if wl.R > 1:
        from token_dispatch_combine_b200 import MoEBalancedRoundTrip, moe_eplb_plan, moe_eplb_remap
        slots = wl.E // wl.R + 1
        plan = moe_eplb_plan(expert_counts, wl.R, slots, device=dev)
        bal = MoEBalancedRoundTrip(wl.T, wl.H, wl.I, wl.E, wl.k, wl.R, slots, dt, device=dev)
        bal.set_plan(plan, wg, wu, wd)
        for _ in range(3):
            bal.forward(x, logits)
        torch.cuda.synchronize()
        before = rt.disp.rank_counts.cpu().numpy().astype(np.float64)
        after = bal.rt.disp.rank_counts.cpu().numpy().astype(np.float64)
        ev_r = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        ev_s = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        for (a, b), (c, d) in zip(ev_r, ev_s):
            flush_and_hold()
            a.record(stream)
            moe_eplb_remap(bal.logical_ids, plan, out=bal.rt.topk_ids)
            b.record(stream)
            flush_and_hold()
            c.record(stream)
            bal.forward(x, logits)
            d.record(stream)
        torch.cuda.synchronize()
        st, bits = moe_get_error()
        if st != 0:
            raise RuntimeError(f"device error word {bits} in the balanced round trip")
        eplb = {
            "physical_experts": plan.P, "slots_per_rank": slots,
            "rank_rows_max_over_mean_static": float(before.max() / before.mean()),
            "rank_rows_max_over_mean_balanced": float(after.max() / after.mean()),
            "remap_us": statistics.median(a.elapsed_time(b) for a, b in ev_r) * 1e3,
            "balanced_step_ms": statistics.median(c.elapsed_time(d) for c, d in ev_s),
            "note": "plan from the warm-up's expert counts; a replica has its expert's weights, so outputs "
                    "are unchanged; on one GPU the ranks are logical, so the balanced step shows only costs: "
                    "the remap and the extra partial GEMM tiles of more (physical) experts",
        }
        del bal
    step_ms, dc_pair_ms, dc_stream_ms, t_disp_rows, t_comb_rows, *stage_max = max_over_ranks(
        [step_ms, dc_pair_ms, dc_stream_ms, *dc_stage, *stage.tolist()], world)
    if router_ms is not None:
        router_ms = max_over_ranks([router_ms], world)[0]

    # End to end through the public API: every step copies its inputs (x, logits) from pinned
    # host memory to the device and its output y back, inside the timed region.
    # MoEHostPipeline overlaps step i's compute with step i+1's upload and step i-1's download.
    # (No L2 flush here: one step touches ~2 GB, far more than the 126 MB L2.)
    from token_dispatch_combine_b200 import MoEHostPipeline
    x_h = torch.from_numpy(x_np.view(np.int16) if x_np.dtype == np.uint16 else x_np).pin_memory()
    l_h = torch.from_numpy(logits_np).pin_memory()
    y_h = torch.empty((wl.T, wl.H), dtype=torch.int16 if dt == torch.bfloat16 else torch.float32).pin_memory()
    pipe = MoEHostPipeline(rt, wg, wu, wd, compute_stream=stream, graphs=args.e2e_graphs == "on")
    pipe.run([(x_h, l_h, y_h)] * max(1, args.warmup))
    torch.cuda.synchronize()
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    torch.cuda._sleep(HOLD_CYCLES * 10)  # let the host enqueue ahead of the GPU
    with ClockSampler(local) as e2e_clocks:
        e_start.record(stream)
        pipe.h2d.wait_stream(stream)
        h0 = time.perf_counter()
        pipe.run([(x_h, l_h, y_h)] * args.steps)
        host_enqueue_ms = (time.perf_counter() - h0) * 1e3 / args.steps  # the host's time to enqueue a step
        e_end.record(pipe.d2h)
        torch.cuda.synchronize()
    barrier(world)
    e2e_ms = e_start.elapsed_time(e_end) / args.steps
    (e2e_ms,) = max_over_ranks([e2e_ms], world)
    # The same steps back to back without the copies (graph replays on the device buffers, no L2
    # flush or hold between steps): what the pipeline's compute alone sustains.
    b2b_ms = None
    if pipe.graphs is not None:
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda._sleep(HOLD_CYCLES * 10)
        g_start, g_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g_start.record(stream)
        with torch.cuda.stream(stream):
            for _ in range(args.steps):
                pipe.graphs[0].replay()
        g_end.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        (b2b_ms,) = max_over_ranks([g_start.elapsed_time(g_end) / args.steps], world)
    # One batch at a time, host in and host out on one stream (no overlap between batches): the
    # latency of a single call sequence through the public API (upload x and logits from pinned
    # memory, the step, download y).
    x_dev1 = torch.empty_like(x)
    l_dev1 = torch.empty_like(logits)
    y_dev1 = torch.empty((wl.T, wl.H), dtype=dt, device=dev)
    lat = []
    for i in range(args.warmup + args.steps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record(stream)
        x_dev1.copy_(x_h.view(dt) if dt == torch.bfloat16 else x_h, non_blocking=True)
        l_dev1.copy_(l_h, non_blocking=True)
        rt.forward(x_dev1, l_dev1, wg, wu, wd, y=y_dev1)
        y_h.copy_(y_dev1.view(y_h.dtype) if y_h.dtype != dt else y_dev1, non_blocking=True)
        b.record(stream)
        torch.cuda.synchronize()
        if i >= args.warmup:
            lat.append(a.elapsed_time(b))
    (single_ms,) = max_over_ranks([statistics.median(lat)], world)
    st, bits = moe_get_error()
    if st != 0:
        raise RuntimeError(f"device error word {bits} during timing")

    if rank != 0:
        return 0
    peaks, peak_src = load_peaks()
    alg = algorithmic(wl)
    t_route, t_disp, t_gu, t_down, t_comb = stage_max
    gemm_tflops = (alg["gateup_flops"] + alg["down_flops"]) / ((t_gu + t_down) * 1e-3) / 1e12
    dc_gbs = (alg["dispatch_bytes"] + alg["combine_bytes"]) / ((t_disp_rows + t_comb_rows) * 1e-3) / 1e9
    # the same with the routing kernel's time and bytes included (it holds the dispatch's counting
    # when route_counts is on)
    rdc_gbs = (alg["route_bytes"] + alg["dispatch_bytes"] + alg["combine_bytes"]) / (
        (t_route + t_disp_rows + t_comb_rows) * 1e-3) / 1e9
    gu_tflops = alg["gateup_flops"] / (t_gu * 1e-3) / 1e12
    peak_tf = peaks["bf16_tflops"]
    tiling = moe_ffn_tiling_for(wl.E, wl.S, FFN_GATE_UP)
    tiling_down = moe_ffn_tiling_for(wl.E, wl.S, FFN_DOWN)
    bounds = gemm_bounds(wl, expert_counts, gather, peaks)
    gu = bounds["gate_up"]
    t_gu_s = t_gu * 1e-3
    if gu["t_hbm"] > gu["t_tensor"]:  # the gate/up launch streams more bytes than its FLOPs need time
        roof_bound, roof_unit, roof_peak = "hbm", "GB/s", peaks["hbm_gbs"]
        roof_achieved = gu["bytes"] / t_gu_s / 1e9
        roof_alg = (f"active gate+up weights + A rows + h = {gu['bytes']:.4g} B "
                    f"(4*S*H*I = {gu['flops']:.4g} FLOP would take {gu['t_tensor'] * 1e6:.0f} us at peak)")
    else:
        roof_bound, roof_unit, roof_peak = "tensor", "TFLOP/s", peak_tf
        roof_achieved = gu_tflops
        roof_alg = f"4*S*H*I = {alg['gateup_flops']:.4g} FLOP"
    gemm_bound_us = (bounds["gate_up"]["t_per_expert"] + bounds["down"]["t_per_expert"]) * 1e6
    cpu = None
    if args.cpu_baseline and world == 1:
        rng = np.random.default_rng(1)
        n_tok, _ = size_oracle_sample(wl, x_np, logits_np, wg_np, wu_np, wd_np, target_s=20.0, rng=rng)
        secs = oracle_sample_step(wl, x_np, logits_np, wg_np, wu_np, wd_np, n_tok, rng)
        cpu = {"value": n_tok / secs, "unit": "tokens/s", "cores": cpu_cores(), "kind": "oracle",
               "sample": f"{n_tok} of {wl.T} tokens through the whole round trip ({secs:.1f} s)"}
    line = {
        "metric": METRIC,
        "value": wl.T * world / (step_ms * 1e-3),
        "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": step_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": wl.dtype, "data": "synthetic",
        "config": config_dict(wl),
        "components": {
            "dispatch_mode": ("index-only dispatch; the gate/up projection gathers its rows from x"
                              if gather else "dispatch moves the rows into x_disp"),
            "route_us": t_route * 1e3, "dispatch_us": t_disp * 1e3, "gate_up_us": t_gu * 1e3,
            "down_us": t_down * 1e3, "combine_us": t_comb * 1e3,
            "dispatch_rows_us": t_disp_rows * 1e3,
            "combine": ("in the down projection's epilogue (moe_ffn_down_combine) + finalize"
                        if rt.combine_in_down else "moe_combine"),
            "dispatch_counting": ("in the routing kernel (moe_route_count; the dispatch kernel scans the chunk "
                                  "counts, permutes and copies)" if rc else "in the dispatch kernel (moe_dispatch)"),
            "route_dispatch_combine_gbs": rdc_gbs, "route_dispatch_combine_frac_hbm": rdc_gbs / peaks["hbm_gbs"],
            "dispatch_combine_gbs": dc_gbs, "dispatch_combine_frac_hbm": dc_gbs / peaks["hbm_gbs"],
            "dispatch_combine_back_to_back_us": dc_pair_ms * 1e3,
            "dispatch_combine_back_to_back_gbs": (alg["dispatch_bytes"] + alg["combine_bytes"]) / (dc_pair_ms * 1e-3) / 1e9,
            "dispatch_combine_back_to_back_frac_hbm":
                (alg["dispatch_bytes"] + alg["combine_bytes"]) / (dc_pair_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
            "dispatch_combine_stream_us": dc_stream_ms * 1e3,
            "dispatch_combine_stream_gbs": (alg["dispatch_bytes"] + alg["combine_bytes"]) / (dc_stream_ms * 1e-3) / 1e9,
            "dispatch_combine_stream_frac_hbm":
                (alg["dispatch_bytes"] + alg["combine_bytes"]) / (dc_stream_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
            "stage_timing": "per-stage CUDA events in a separate pass of the same steps (each stage boundary "
                            "adds event overhead); back_to_back: one event pair around dispatch+combine; stream: 20 dispatch+combine pairs over 4 buffer sets (>L2) under one event pair",
            "grouped_gemm_tflops": gemm_tflops, "grouped_gemm_frac_bf16": gemm_tflops / peak_tf,
            "grouped_gemm_bound_us": gemm_bound_us,
            "grouped_gemm_frac_of_bound": gemm_bound_us / ((t_gu + t_down) * 1e3),
            "grouped_gemm_bound": "sum over experts of max(FLOPs / bf16 peak, bytes / HBM peak), both "
                                  "projections, from this layer's expert counts",
            **({} if router_ms is None else {
                "router_topk_us": router_ms * 1e3,
                "router_topk_gbs": alg["router_bytes"] / (router_ms * 1e-3) / 1e9,
                "router_topk_frac_hbm": alg["router_bytes"] / (router_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                "router_topk_timing": "moe_router_topk (logits = x W_r^T + bias, then top-k), L2 flushed, "
                                      "events per call; bytes T*H*2 + E*H*2 + T*k*8"}),
            **({} if eplb is None else {"eplb": eplb}),
            **({} if masked is None else {"masking_form": masked}),
            **({} if ep_info is None else {"exchange_between_ranks_one_gpu": ep_info}),
            "graph_replay_ms": graph_ms,
            **({} if graph_err is None else {"graph_replay_error": graph_err}),
            "ffn_tiling": {"gate_up": "pair" if tiling == FFN_TILING_PAIR else "single",
                           "down": "pair" if tiling_down == FFN_TILING_PAIR else "single"},
        },
        "roofline": {
            "kernel": ("grouped_gemm_tc2_kernel<gate/up, SwiGLU epilogue" + (", rows gathered from x" if gather else "")
                       + "> (256-row tiles on 2-SM clusters)"
                       if tiling == FFN_TILING_PAIR else
                       "grouped_gemm_tc_kernel<gate/up, SwiGLU epilogue" + (", rows gathered from x" if gather else "")
                       + "> (128-row tiles)"),
            "bound": roof_bound, "achieved": roof_achieved, "peak": roof_peak, "unit": roof_unit,
            "frac": roof_achieved / roof_peak, "traffic": dram_traffic(wl.name, gather),
            "peak_source": f"{peak_src} " + ("bf16 dense (burst)" if roof_bound == "tensor" else "HBM copy"),
            "algorithmic_per_launch": roof_alg,
        },
        "e2e": {"value": wl.T * world / (e2e_ms * 1e-3), "unit": "tokens/s",
                "h2d_bytes_per_step": int(x_np.nbytes + logits_np.nbytes), "d2h_bytes_per_step": int(y_h.numel() * y_h.element_size()),
                "api": "MoEHostPipeline (upload, compute and download of consecutive steps overlap"
                       + ("; each step one CUDA graph replay)" if args.e2e_graphs == "on" else "; eager calls)"),
                "host_enqueue_ms_per_step": host_enqueue_ms,
                "compute_back_to_back_ms": b2b_ms,
                "compute_back_to_back": "the same steps' graph replays back to back with no copies, no L2 flush "
                                        "and no hold between them",
                "clocks": e2e_clocks.summary(),
                "single_batch_ms": single_ms,
                "single_batch": "one batch host to host on one stream (upload x and logits, MoERoundTrip.forward, "
                                "download y), no overlap with other batches; median of the steps"},
        "gpu_launches": MoERoundTrip.KERNELS_PER_FORWARD * args.steps,  # kernels of this library in the timed region
        "clocks": clocks.summary(),
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="gptoss_uniform", choices=sorted(synth.WORKLOADS) + sorted(synth.PROFILE_WORKLOADS),
                    help="benchmark layer (or a profiling case: a small layer of the same shapes)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ffn-tiling", default="auto", choices=["auto", "single", "pair"],
                    help="tile shape of the bf16 expert FFN (moe_set_ffn_tiling); auto picks by rows per expert")
    ap.add_argument("--dispatch", default="auto", choices=["auto", "rows", "gather"],
                    help="rows: dispatch writes x_disp; gather: index-only dispatch, the gate/up projection "
                         "gathers its rows from x (moe_ffn_gate_up_gather); auto: MoERoundTrip's choice")
    ap.add_argument("--route-counts", default="on", choices=["on", "off"],
                    help="on: the routing kernel also does the dispatch's counting (moe_route_count + "
                         "moe_dispatch_counted); off: moe_route + moe_dispatch")
    ap.add_argument("--combine-in-down", default="off", choices=["on", "off"],
                    help="on: the down projection's epilogue does the combine (moe_ffn_down_combine, float32 "
                         "atomics into a [T, H] accumulator) and a finalize kernel rounds it into y")
    ap.add_argument("--e2e-graphs", default="on", choices=["on", "off"],
                    help="on: the end-to-end pipeline replays one captured CUDA graph per step")
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false",
                    help="skip the CPU oracle leg (used for profiler runs)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    wl = synth.WORKLOADS.get(args.config) or synth.PROFILE_WORKLOADS[args.config]
    if args.impl == "reference":
        return run_reference(args, wl)
    rc = run_ours(args, wl)
    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return rc


if __name__ == "__main__":
    sys.exit(main())
