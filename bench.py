#!/usr/bin/env python
"""Benchmark of the quantized-state decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload gdn|mamba2|gla|stack24|tiny-gdn]

One "step" advances the workload's batch by one token under each of its
arms.  The default workload is the largest, the 24-layer gated delta-rule
stack (12288 tiles of Dk = Dv = 128, readout every step) under its two arms,
INT4 G32 persistent + BDR and INT8 G32 dynamic: one kernel launch each.  The
metric is decode steps/s (whole job; N GPUs run independent shards, so
scaling is weak) and the algorithmic state traffic in GB/s as a fraction of
the measured HBM peak; the roofline line reports the quantized-state arm
furthest from that peak.

L2 residency: an arm's state can be smaller than B200's L2, so each arm's
steps rotate over G independent request groups whose states together exceed
2x the L2 size (G chosen per arm, since the arms are timed one after the
other); step t uses group t mod G and pool slot t mod P of the inputs.  No
state or input is therefore warm in L2 when its step runs.

Timing: W untimed warm-up steps per arm (eager), then every CUDA graph the
timed region replays (a full cycle of P steps and the K mod P tail) is
replayed once, the states are re-initialized, and each arm's K steps are
replayed from those graphs, bracketed by CUDA events on the launching
stream, with a barrier and a device synchronize on both sides; the max over
ranks is reported.  Between the synchronize and the first timed event the
stream writes a buffer twice the L2 size (clearing L2 and keeping the GPU
busy up to the timed region).  SM clocks and throttle reasons are sampled
through NVML during the timed region.

The `e2e` figure runs the same steps through the public API with host
buffers: each step copies its inputs from pinned host memory, launches the
arms and copies the readouts back, all inside the timed region.

`--impl reference` times the CPU oracle (the plain C implementation used
as the correctness reference) on the host cores on a bounded sample of
tiles per step, reported in the same unit.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from ssm_decode_step_b200 import workloads as W  # noqa: E402

PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
FALLBACK_HBM_GBS = 6650.0


# ---------------------------------------------------------------------------
# bytes per launch (algorithmic)
# ---------------------------------------------------------------------------

def arm_bytes(w: W.Workload, arm: W.Arm, readout: bool = True) -> int:
    """Algorithmic bytes one decode-step launch must move: codes read and
    written, scales read (and written unless persistent), q, k, v, alpha,
    beta read, o written, and the FP32 shadow read and written (yoked)."""
    T, dk, dv = w.tiles, w.dk, w.dv
    codes = T * dv * dk * arm.bits // 8
    scales = T * dv * (dk // arm.group) * 4
    alpha = T * (dk if w.decay == "diagonal" else 1) * 4
    inputs = T * ((dk if readout else 0) + dk + dv) * 4 + alpha + T * 4
    out = T * dv * 4 if readout else 0
    b = 2 * codes + scales * (1 if arm.policy == "persistent" else 2) + inputs + out
    if arm.policy == "yoked":
        b += 2 * T * dv * dk * 4
    return b


def state_bytes(w: W.Workload, arm: W.Arm) -> int:
    T, dk, dv = w.tiles, w.dk, w.dv
    b = T * dv * dk * arm.bits // 8 + T * dv * (dk // arm.group) * 4
    if arm.policy == "yoked":
        b += T * dv * dk * 4
    return b


# The sources the decode-step kernel is compiled from: a committed traffic
# figure stays valid while none of them, nor the nvcc flags, changes.
STEP_SOURCES = ("qstate_step.cuh", "qstate_stream.cuh", "qstate_kernels.cuh", "qstate_launch.h",
                "qstate_launch_impl.cuh", "inst_b4_d128.cu", "inst_b4_d64.cu", "inst_b8_d128.cu",
                "inst_b8_d64.cu")


def source_sha() -> str:
    h = hashlib.sha256()
    pkg = os.path.join(ROOT, "ssm_decode_step_b200")
    for f in STEP_SOURCES:
        with open(os.path.join(pkg, "csrc", f), "rb") as fh:
            h.update(f.encode() + fh.read())
    from ssm_decode_step_b200 import build as B
    h.update(B.flags_key().encode())
    return h.hexdigest()[:16]


def load_peak():
    try:
        with open(PEAKS_FILE) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def load_traffic(kernel_key: str):
    """DRAM bytes per launch from a committed ncu capture, if the kernel
    sources have not changed since it was taken."""
    try:
        with open(TRAFFIC_FILE) as f:
            data = json.load(f)
        ent = data.get(kernel_key)
        if ent and ent.get("source_sha") == source_sha():
            return ent["dram_bytes_per_launch"]
    except Exception:
        pass
    return None


# ---------------------------------------------------------------------------
# clocks
# ---------------------------------------------------------------------------

REASON_BITS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML on a thread."""

    def __init__(self, torch_device_index: int, period_s: float = 0.005):
        self.samples = []
        self.max_mhz = None
        self.period = period_s
        self._stop = threading.Event()
        self._thr = None
        self.h = None
        try:
            import pynvml as N
            N.nvmlInit()
            self.N = N
            import torch
            props = torch.cuda.get_device_properties(torch_device_index)
            bus = getattr(props, "pci_bus_id", None)
            dom = getattr(props, "pci_domain_id", 0)
            dev = getattr(props, "pci_device_id", 0)
            if bus is not None:
                busid = "%08x:%02x:%02x.0" % (dom, bus, dev)
                self.h = N.nvmlDeviceGetHandleByPciBusId(busid.encode())
            else:
                self.h = N.nvmlDeviceGetHandleByIndex(torch_device_index)
            self.max_mhz = N.nvmlDeviceGetMaxClockInfo(self.h, N.NVML_CLOCK_SM)
        except Exception:
            self.h = None

    def _reasons(self):
        N = self.N
        for fn in ("nvmlDeviceGetCurrentClocksEventReasons", "nvmlDeviceGetCurrentClocksThrottleReasons"):
            if hasattr(N, fn):
                return getattr(N, fn)(self.h)
        return 0

    def _run(self):
        N = self.N
        while not self._stop.is_set():
            try:
                self.samples.append((N.nvmlDeviceGetClockInfo(self.h, N.NVML_CLOCK_SM), self._reasons()))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.h is not None:
            self._thr = threading.Thread(target=self._run, daemon=True)
            self._thr.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thr is not None:
            self._thr.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mhz = [m for m, _ in self.samples]
        mask = 0
        for _, r in self.samples:
            mask |= int(r)
        reasons = [name for bit, name in REASON_BITS.items() if mask & bit and name != "gpu_idle"]
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# distributed plumbing (barrier and max over ranks only; no data-path collective)
# ---------------------------------------------------------------------------

def pool_slots(w: W.Workload, l2: int) -> int:
    """Input slots: enough that the pool exceeds twice the L2 size (so no
    step finds its inputs in L2), a power of two from 16 to 64."""
    per_slot = w.tiles * (2 * w.dk + w.dv + (w.dk if w.decay == "diagonal" else 1) + 1) * 4
    P = 16
    while P < 64 and P * per_slot < 2 * l2:
        P *= 2
    return P


def l2_flush(dev, l2: int):
    """A device buffer of twice the L2 size, written (on the current stream)
    between the last synchronize and the first timed event."""
    import torch
    return torch.empty(2 * l2 // 4, dtype=torch.float32, device=dev)


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def dist_init(ws, backend):
    if ws <= 1:
        return None
    import datetime
    import torch.distributed as dist
    dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(dist, values, device):
    if dist is None:
        return values
    import torch
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


# ---------------------------------------------------------------------------
# CPU baseline: the oracle as it stands, on a bounded sample of tiles
# ---------------------------------------------------------------------------

def oracle_sample_rate(w: W.Workload, budget_s: float, steps: int = 0, max_tiles: int = 256):
    """Oracle steps/s on the host cores, measured on a seeded sample of tiles
    and scaled to whole steps (tiles are independent, so time is linear in
    the number of tiles).  With `steps` given, exactly that many steps run and
    the sample is sized to take about budget_s; otherwise max_tiles tiles run
    for as many steps as fill about budget_s."""
    from oracle import oracle as O
    rng = np.random.default_rng(12345)
    threads = O.num_threads()

    def make(n):
        tiles = np.sort(rng.choice(w.tiles, size=n, replace=False))
        S0 = W.initial_state(w, tiles)
        sts = []
        for arm in w.arms:
            cfg = O.OracleConfig(n, w.dk, w.dv, arm.bits, arm.group, w.delta, w.decay, arm.policy,
                                 arm.rounding)
            sts.append(O.init(cfg, S0))
        return tiles, sts

    # calibration: one step of a small sample (untimed warm-up of the oracle)
    n0 = min(w.tiles, max(threads, 16))
    tiles, sts = make(n0)
    inp = W.slot(w, 0, tiles)
    t0 = time.perf_counter()
    for st in sts:
        O.step(st, *inp, want_o=w.readout)
    per_tile_step = max(time.perf_counter() - t0, 1e-6) / n0
    if steps:
        n = int(budget_s / (per_tile_step * steps))
        n = max(min(threads, w.tiles), min(n, max_tiles, w.tiles))
    else:
        n = min(max_tiles, w.tiles)
        steps = int(budget_s / (per_tile_step * n))
        steps = max(2, min(steps, 100000))
    tiles, sts = make(n)
    P = min(steps, 16)
    pool = [W.slot(w, t, tiles) for t in range(P)]
    t0 = time.perf_counter()
    for t in range(steps):
        inp = pool[t % P]
        for st in sts:
            O.step(st, *inp, want_o=w.readout)
    dt = time.perf_counter() - t0
    rate = (n / w.tiles) * steps / dt
    sample = (f"{n} of {w.tiles} tiles (seeded random sample), {steps} steps, all {len(w.arms)} arms; "
              f"steps/s scaled by {w.tiles}/{n}")
    return rate, threads, sample, dt


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def run_ours(args):
    import torch

    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = dist_init(ws, "nccl")

    from ssm_decode_step_b200 import Config, QState, qstate as Q
    Q.lib()
    # N GPUs split one workload: rank r owns the contiguous tile range
    # [r T / N, (r + 1) T / N) (tiles are independent; no exchange)
    w_all = W.get(args.workload)
    w = W.shard(w_all, rank, ws) if ws > 1 else w_all
    arms = list(w.arms)
    K, Wm = args.steps, args.warmup
    readout = w.readout

    # input pool on the device: P slots of (q, k, v, alpha, beta)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    P = args.pool or pool_slots(w, l2)
    args.pool = P
    host = W.pool(w, P)
    pool = [torch.from_numpy(a).to(dev) for a in host]

    # request groups so that all groups' states exceed 2x L2
    pool_bytes = P * sum(a[0].nbytes for a in host)

    def groups_for(arm):
        G = args.groups or max(1, -(-2 * l2 // state_bytes(w, arm)))
        G = min(G, P)            # every group needs its own input slots in the cycle
        while P % G:             # the captured cycle of P steps visits each group equally
            G -= 1
        return G

    groups = [groups_for(a) for a in arms]
    l2_resident = [g * state_bytes(w, a) + pool_bytes < 2 * l2 for g, a in zip(groups, arms)]
    S0 = torch.from_numpy(W.initial_state(w)).to(dev)

    cfgs = [Config(w.tiles, w.dk, w.dv, a.bits, a.group, w.delta, w.decay, a.policy, a.rounding)
            for a in arms]
    states = [[QState(c, dev) for _ in range(g)] for c, g in zip(cfgs, groups)]
    outs = [torch.empty((w.tiles, w.dv), dtype=torch.float32, device=dev) if readout else None
            for _ in arms]

    def reinit():
        for ai, c in enumerate(cfgs):
            for st in states[ai]:
                st.init(S0)

    def launch(ai, t):
        s = t % P
        st = states[ai][t % len(states[ai])]
        st.step(pool[0][s], pool[1][s], pool[2][s], pool[3][s], pool[4][s], outs[ai])

    stream = torch.cuda.Stream(device=dev)
    reinit()
    torch.cuda.synchronize()
    # warm-up, eager
    with torch.cuda.stream(stream):
        for t in range(Wm):
            for ai in range(len(arms)):
                launch(ai, t)
    stream.synchronize()

    # graphs of P steps per arm (one full cycle of groups and slots), and a tail
    n_main, tail = divmod(K, P)

    def capture(ai, nsteps):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for t in range(nsteps):
                launch(ai, t)
        return g

    graphs = [capture(ai, P) for ai in range(len(arms))]
    tails = [capture(ai, tail) if tail else None for ai in range(len(arms))]
    # warm every graph the timed region replays (the first replay of a graph
    # uploads it), then restart every state from S0
    with torch.cuda.stream(stream):
        for ai in range(len(arms)):
            graphs[ai].replay()
            if tails[ai] is not None:
                tails[ai].replay()
    stream.synchronize()
    reinit()
    torch.cuda.synchronize()
    flush = l2_flush(dev, l2)

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in arms]
    sampler = ClockSampler(local)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with sampler:
        with torch.cuda.stream(stream):
            flush.fill_(1.0)
            flush.fill_(2.0)
            for ai in range(len(arms)):
                ev[ai][0].record(stream)
                for _ in range(n_main):
                    graphs[ai].replay()
                if tails[ai] is not None:
                    tails[ai].replay()
                ev[ai][1].record(stream)
        stream.synchronize()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    del flush
    arm_ms = [a.elapsed_time(b) for a, b in ev]
    arm_ms = max_over_ranks(dist, arm_ms, dev)
    total_ms = sum(arm_ms)
    clocks = sampler.summary()
    fp32 = None if args.no_fp32 else run_fp32_state(args, w, dev, stream, dist, pool, host, S0, l2,
                                                   pool_bytes)
    plain_us = {a.name: arm_ms[i] * 1e3 / K for i, a in enumerate(arms)}
    lrb = None if args.lrb_rank <= 1 else run_lrb(args, w, dev, stream, dist, pool, S0, l2,
                                                   pool_bytes, plain_us)

    # ---- end to end through the public API with host buffers
    e2e = run_e2e(args, w, arms, cfgs, states, dev, stream, dist, host, reinit)

    peak, peak_src = load_peak()
    # whole-job rates: every step advances all ranks' shards, i.e. the whole
    # workload, and the slowest rank's time is the step time
    bytes_step = sum(arm_bytes(w_all, a, readout) for a in arms)
    value = K / (total_ms / 1e3)
    gbs = bytes_step * K / (total_ms / 1e3) / 1e9
    # the roofline line: the quantized-state arm furthest from the HBM peak
    # (the yoked arm moves mostly its FP32 shadow and is reported per arm)
    quant = [i for i, a in enumerate(arms) if a.policy != "yoked"] or list(range(len(arms)))
    fracs = {i: arm_bytes(w, arms[i], readout) / (arm_ms[i] / 1e3 / K) / 1e9 / peak for i in quant}
    dom = min(fracs, key=fracs.get)
    dom_bytes = arm_bytes(w, arms[dom], readout)      # per GPU (this rank's shard)
    dom_s = arm_ms[dom] / 1e3 / K
    achieved = dom_bytes / dom_s / 1e9
    kernel_key = f"{w.name}:{arms[dom].name}"
    traffic = load_traffic(kernel_key)
    per_arm = {}
    for ai, a in enumerate(arms):
        s = arm_ms[ai] / 1e3 / K
        b = arm_bytes(w, a, readout)
        per_arm[a.name] = {"us_per_launch": round(s * 1e6, 3), "bytes_per_launch": b,
                           "gbs": round(b / s / 1e9, 1), "frac": round(b / s / 1e9 / peak, 4),
                           "traffic": load_traffic(f"{w.name}:{a.name}")}

    line = {
        "metric": "quantized-state decode steps/sec; state GB/s as fraction of B200 HBM peak",
        "value": round(value, 2),
        "unit": "steps/s",
        "n_gpus": ws,
        "steps": K,
        "warmup": Wm,
        "ms_per_step": round(total_ms / K, 6),
        "higher_is_better": True,
        "scaling": "strong",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic (seeded; shapes and value laws of the workload)",
        "config": {
            "workload": f"{w_all.name}: {w_all.description}",
            "tiles": w_all.tiles,
            "tiles_per_gpu": w.tiles,
            "step": f"one token for all {w.tiles} tiles under each arm ({len(arms)} launches)",
            "arms": [a.name for a in arms],
            "readout": readout,
            "l2": "; ".join(
                (f"{a.name}: L2-resident ({g} groups x {state_bytes(w, a) / 1e6:.3f} MB state, "
                 f"smaller than L2)" if res else
                 f"{a.name}: inputs larger than L2 ({g} request groups x "
                 f"{state_bytes(w, a) / 1e6:.1f} MB state + {pool_bytes / 1e6:.0f} MB of input "
                 f"slots rotated; L2 {l2 / 1e6:.0f} MB)")
                for a, g, res in zip(arms, groups, l2_resident)),
            "parallelism": (f"tile shards on {ws} GPU(s): rank r owns tiles [r*T/N, (r+1)*T/N) of the "
                            f"one workload; no collective on the step"),
        },
        "state_gbs": round(gbs, 1),
        "state_frac": round(gbs / peak, 4),
        "arms": per_arm,
        "roofline": {
            "bound": "hbm",
            "kernel": f"{'stream_step_kernel' if arms[dom].policy != 'yoked' else 'step_kernel'} "
                      f"({kernel_key}; the quantized-state arm furthest from the peak)",
            "quantized_arms_frac": {arms[i].name: round(f, 4) for i, f in fracs.items()},
            "achieved": round(achieved, 1),
            "peak": peak,
            "peak_source": peak_src,
            "unit": "GB/s",
            "frac": round(achieved / peak, 4),
            "traffic": traffic,
            "algorithmic_bytes_per_launch": dom_bytes,
        },
        "e2e": e2e,
        "fp32_state": fp32 and dict(fp32, **{
            "quantized_speedup": {a.name: round(fp32["us_per_launch"] / (arm_ms[i] * 1e3 / K), 3)
                                  for i, a in enumerate(arms)},
            "state_memory_ratio": {a.name: round(w.tiles * w.dv * w.dk * 4 / state_bytes(w, a), 3)
                                   for a in arms}}),
        "lrb": lrb,
        "gpu_launches": ws * K * len(arms),
        "clocks": clocks,
    }
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        rate, threads, sample, dt = oracle_sample_rate(w, budget_s=args.cpu_budget)
        line["cpu_baseline"] = {"value": round(rate, 4), "unit": "steps/s", "cores": threads,
                                "kind": "oracle", "sample": sample, "seconds": round(dt, 2)}
    if rank == 0:
        print(json.dumps(line), flush=True)
    for g in graphs + [t for t in tails if t is not None]:
        del g
    if dist is not None:
        dist.destroy_process_group()


def fp32_bytes(w: W.Workload, readout: bool = True) -> int:
    T, dk, dv = w.tiles, w.dk, w.dv
    alpha = T * (dk if w.decay == "diagonal" else 1) * 4
    return 2 * T * dv * dk * 4 + T * ((dk if readout else 0) + dk + dv) * 4 + alpha + T * 4 + \
        (T * dv * 4 if readout else 0)


def run_fp32_state(args, w, dev, stream, dist, pool, host, S0, l2, pool_bytes):
    """The same steps on an FP32 state (qstate_fp32_decode_step): the
    baseline of the quantized arms, timed the same way (CUDA graphs, events,
    request groups sized past 2x L2).  Not part of the step."""
    import torch
    from ssm_decode_step_b200 import Config, qstate as Q
    K, P = args.steps, args.pool
    cfg = Config(w.tiles, w.dk, w.dv, 8, 32, w.delta, w.decay)
    sb = w.tiles * w.dv * w.dk * 4
    G = max(1, -(-2 * l2 // sb))
    G = min(G, P)
    while P % G:
        G -= 1
    states = [S0.clone() for _ in range(G)]
    o = torch.empty((w.tiles, w.dv), dtype=torch.float32, device=dev) if w.readout else None

    def launch(t):
        s = t % P
        Q.fp32_decode_step(cfg, states[t % G], pool[0][s], pool[1][s], pool[2][s], pool[3][s],
                           pool[4][s], o, stream)

    with torch.cuda.stream(stream):
        for t in range(args.warmup):
            launch(t)
    stream.synchronize()
    n_main, tail = divmod(K, P)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for t in range(P):
            launch(t)
    gt = None
    if tail:
        gt = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gt, stream=stream):
            for t in range(tail):
                launch(t)
    with torch.cuda.stream(stream):
        g.replay()
    stream.synchronize()
    for st in states:
        st.copy_(S0)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(n_main):
            g.replay()
        if gt is not None:
            gt.replay()
        e1.record(stream)
    stream.synchronize()
    ms = max_over_ranks(dist, [e0.elapsed_time(e1)], dev)[0]
    del g, gt
    peak, _ = load_peak()
    b = fp32_bytes(w, w.readout)
    s = ms / 1e3 / K
    return {"us_per_launch": round(s * 1e6, 3), "bytes_per_launch": b,
            "gbs": round(b / s / 1e9, 1), "frac": round(b / s / 1e9 / peak, 4),
            "l2": f"{G} request groups x {sb / 1e6:.1f} MB FP32 state + {pool_bytes / 1e6:.0f} MB inputs"}


def lrb_bytes(w: W.Workload, arm: W.Arm, rank: int, slot: int, readout: bool = True) -> int:
    """Algorithmic bytes of one Low-Rank Bypass step at position `slot` of
    its period: the stored state is read at every step and written only at
    the merge; the accumulated decay and the buffered keys are read (and
    written at bypass steps), the coefficients read for slots < slot and
    written for the slot."""
    T, dk, dv = w.tiles, w.dk, w.dv
    merge = slot == rank - 1
    codes = T * dv * dk * arm.bits // 8
    scales = T * dv * (dk // arm.group) * 4
    b = codes + scales
    if merge:
        b += codes + (scales if arm.policy != "persistent" else 0)
    b += T * (2 * dk + dv + 2) * 4 + (T * dk * 4 if w.decay == "diagonal" else 0)
    b += T * dv * 4 if readout else 0
    b += (T * dk * 4 if slot > 0 else 0) + (0 if merge else T * dk * 4)      # A in / out
    b += T * slot * dk * 4 + (0 if merge else T * (slot + 1) * dk * 4)      # K in / out
    b += T * dv * slot * 4 + (0 if merge else T * dv * 4)                    # U read / write
    if arm.policy == "yoked":
        b += 2 * T * dv * dk * 4
    return b


def run_lrb(args, w, dev, stream, dist, pool, S0, l2, pool_bytes, plain_us):
    """Every arm of the workload again with Low-Rank Bypass of rank R
    (qstate_lrb_decode_step): R - 1 bypass steps and one merge per period,
    timed over whole periods the same way as the arms (CUDA graphs, events,
    request groups past 2x L2).  Reported per step, averaged over the period.
    Not part of the step."""
    import torch
    from ssm_decode_step_b200 import Config, QState, qstate as Q
    R, P = args.lrb_rank, args.pool
    out = {"rank": R}
    peak, _ = load_peak()
    for arm in w.arms:
        cfg = Config(w.tiles, w.dk, w.dv, arm.bits, arm.group, w.delta, w.decay, arm.policy,
                     arm.rounding)
        a_b, k_b, u_b = Q.lrb_query_sizes(cfg, R)
        gb = state_bytes(w, arm) + 2 * a_b + 2 * k_b + u_b
        G = max(1, -(-2 * l2 // gb))
        groups = []
        for _ in range(G):
            st = QState(cfg, dev).init(S0)
            groups.append((st, Q.LrbBuffers(cfg, R, dev)))
        o = torch.empty((w.tiles, w.dv), dtype=torch.float32, device=dev) if w.readout else None
        # one graph = one period of every group; inputs keep cycling the pool
        order = [(gi, slot) for slot in range(R) for gi in range(G)]

        def launch(t, gi, slot):
            st, b = groups[gi]
            i = slot % 2
            sl = t % P
            Q.lrb_decode_step(cfg, R, slot, st.codes, st.scales, st.shadow, b.A[i], b.A[1 - i],
                              b.K[i], b.K[1 - i], b.U, pool[0][sl], pool[1][sl], pool[2][sl],
                              pool[3][sl], pool[4][sl], o, stream)

        with torch.cuda.stream(stream):
            for t, (gi, slot) in enumerate(order):
                launch(t, gi, slot)
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for t, (gi, slot) in enumerate(order):
                launch(t, gi, slot)
        reps = max(1, args.steps // len(order))
        for st, _ in groups:
            st.init(S0)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if dist is not None:
            dist.barrier()
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(reps):
                g.replay()
            e1.record(stream)
        stream.synchronize()
        ms = max_over_ranks(dist, [e0.elapsed_time(e1)], dev)[0]
        del g
        steps = reps * len(order)
        sec = ms / 1e3 / steps
        b = sum(lrb_bytes(w, arm, R, sl, w.readout) for sl in range(R)) / R
        out[arm.name] = {"us_per_step": round(sec * 1e6, 3), "bytes_per_step": int(b),
                         "gbs": round(b / sec / 1e9, 1), "frac": round(b / sec / 1e9 / peak, 4),
                         "speedup_vs_plain": round(plain_us[arm.name] / (sec * 1e6), 3),
                         "l2": f"{G} request groups x {gb / 1e6:.1f} MB (state + buffers)",
                         "steps": steps}
        del groups
        torch.cuda.empty_cache()
    return out


def run_e2e(args, w, arms, cfgs, states, dev, stream, dist, host, reinit):
    """Same steps through the library's host-buffer pipeline
    (qstate_pipeline_step, one C call per step): per step, the packed inputs
    are copied up from pinned host memory, every arm's step runs, and the
    readouts are copied back to pinned host memory; all inside the timed
    region.  The copies run on the pipeline's own streams, four steps deep,
    so step t's inputs go up and step t-1's readouts come down while the
    state updates run in order on the compute stream."""
    import math
    import torch
    from ssm_decode_step_b200 import HostPipeline

    K = min(args.steps, args.e2e_steps)
    P = args.pool
    T = w.tiles
    # one packed pinned buffer per slot: q | k | v | alpha | beta
    parts = [np.ascontiguousarray(a) for a in host]
    sizes = [a[0].size for a in parts]
    packed = torch.empty((P, sum(sizes)), dtype=torch.float32).pin_memory()
    for s in range(P):
        packed[s] = torch.from_numpy(np.concatenate([a[s].reshape(-1) for a in parts]))
    readout = w.readout
    o_host = torch.empty((P, len(arms), T, w.dv), dtype=torch.float32).pin_memory()
    slots_in = [packed[s] for s in range(P)]
    slots_out = [o_host[s] if readout else None for s in range(P)]
    # the request group each arm steps at step t (the cycle repeats every `period` steps)
    period = math.lcm(*[len(g) for g in states])
    combos = [tuple(g[t % len(g)] for g in states) for t in range(period)]
    pl = HostPipeline(combos[0], depth=4)

    def one(t):
        pl.step(slots_in[t % P], slots_out[t % P], stream, combos[t % period])

    # warm-up: one full cycle of the pinned slots (the first transfer to or
    # from a page-locked page costs more than later ones, as in any serving
    # loop that reuses its staging buffers)
    reinit()
    for t in range(max(3, args.warmup, P)):
        one(t)
    pl.sync()
    reinit()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    pl.wait_stream(stream)
    for t in range(K):
        one(t)
    pl.join(stream)
    e1.record(stream)
    torch.cuda.synchronize()
    pl.close()
    ms = max_over_ranks(dist, [e0.elapsed_time(e1)], dev)[0]
    # each rank pipelines its shard: a step of every rank is one whole-workload step
    return {"value": round(K / (ms / 1e3), 2), "unit": "steps/s",
            "h2d_bytes_per_step": int(sum(sizes) * 4),
            "d2h_bytes_per_step": int(len(arms) * T * w.dv * 4) if readout else 0,
            "steps": K,
            "pipelining": "qstate_pipeline_step: inputs up / readouts down on the pipeline's "
                          "own streams, four buffers"}


# ---------------------------------------------------------------------------
# reference arm: the CPU oracle
# ---------------------------------------------------------------------------

def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return
    w = W.get(args.workload)
    from oracle import oracle as O
    # warm-up on a single tile (untimed), then the timed steps on a sample
    rate, threads, sample, dt = oracle_sample_rate(w, budget_s=args.ref_budget, steps=args.steps)
    peak, _ = load_peak()
    bytes_step = sum(arm_bytes(w, a, w.readout) for a in w.arms)
    line = {
        "impl": "reference",
        "metric": "quantized-state decode steps/sec; state GB/s as fraction of B200 HBM peak",
        "value": round(rate, 4),
        "unit": "steps/s",
        "n_gpus": ws,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(1e3 / rate, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic (seeded; shapes and value laws of the workload)",
        "config": {"workload": w.description, "tiles": w.tiles,
                   "step": f"one token for all {w.tiles} tiles under each arm ({len(w.arms)} arms)",
                   "arms": [a.name for a in w.arms]},
        "state_gbs": round(bytes_step * rate / 1e9, 3),
        "cpu_baseline": {"value": round(rate, 4), "unit": "steps/s", "cores": threads,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(rate, 4), "unit": "steps/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# recall over a decode horizon (a measurement of the quantized recurrence,
# not a throughput figure)
# ---------------------------------------------------------------------------
def plant(S_w: np.ndarray, kstar: np.ndarray, vstar: np.ndarray) -> np.ndarray:
    """S0 that maps the unit key k* to v* and agrees with S_w on the
    complement of k*: S0 = S_w + (v* - S_w k*) k*^T, in float64 on the host,
    rounded once to float32 (the probe the horizon measurement reads back)."""
    S = S_w.astype(np.float64)
    k = kstar.astype(np.float64)
    v = vstar.astype(np.float64)
    S += np.einsum("ti,tj->tij", v - np.einsum("tij,tj->ti", S, k), k)
    return np.ascontiguousarray(S, dtype=np.float32)


def run_recall(args):
    """Plant (k*, v*) in S0, decode H distractor steps under every arm (and,
    with --recall-lrb R, the same arms with Low-Rank Bypass of rank R) and
    the FP32 state, and read the fact back at power-of-two checkpoints
    ("When Dynamic Scaling Fails": recall of a fact planted before
    quantization began, as the decode horizon grows; the scale-state
    feedback shows as norm inflation).  The read is each step's own readout
    with q = k*: o_t = S_t k* from the updated state (for a Low-Rank Bypass
    arm, the stored state with its accumulated decay plus the buffer).  The
    state norm is that of the stored state (qstate_state_sq_norms); for a
    bypass arm it is taken at the ends of periods only, where the buffer has
    just been merged.  Prints one JSON line."""
    import torch
    from ssm_decode_step_b200 import qstate as Q
    w = W.get("recall")
    H, T, dk, dv = args.recall_steps, w.tiles, w.dk, w.dv
    dev = torch.device("cuda")
    torch.cuda.set_device(0)
    kstar, vstar = W.probe(w)
    S0 = plant(W.initial_state(w), kstar, vstar)
    P = max(1, min(args.pool or 64, H))
    pool = [torch.from_numpy(a).to(dev) for a in W.pool(w, P)]
    kst = torch.from_numpy(kstar).to(dev)
    zk = torch.zeros((T, dk), dtype=torch.float32, device=dev)
    zv = torch.zeros((T, dv), dtype=torch.float32, device=dev)
    one = torch.ones(T, dtype=torch.float32, device=dev)
    zero = torch.zeros(T, dtype=torch.float32, device=dev)
    o = torch.empty((T, dv), dtype=torch.float32, device=dev)
    nrm = torch.empty(T, dtype=torch.float64, device=dev)
    marks = sorted({0, H} | {1 << i for i in range(40) if (1 << i) <= H})
    launches = 0

    def trajectory(step, probe0, norms_at):
        """step(t, want_o) advances one step (readout into o with q = k* when
        want_o); probe0() reads the state before the first step."""
        nonlocal launches
        rec, norms = [], []
        t = 0
        for m in marks:
            if m == 0:
                probe0()
                launches += 2
            while t < m:
                t += 1
                step(t - 1, t == m)
                launches += 1
            if m > 0:
                if norms_at(m):
                    norms_at(m)(nrm)
                    launches += 1
                else:
                    nrm.fill_(float("nan"))
            torch.cuda.synchronize()
            rec.append(o.cpu().numpy().astype(np.float64))
            norms.append(nrm.cpu().numpy())
        return np.stack(rec), np.stack(norms)

    t0 = time.time()
    cfg32 = Q.Config(T, dk, dv, 8, 32, w.delta, w.decay)
    S = torch.from_numpy(S0.copy()).to(dev)
    fp = trajectory(
        lambda i, want: Q.fp32_decode_step(cfg32, S, kst, pool[1][i % P], pool[2][i % P],
                                           pool[3][i % P], pool[4][i % P], o if want else None),
        # before the first step: a zero update (alpha = 1, k = 0, beta = 0) leaves S unchanged
        lambda: (Q.fp32_decode_step(cfg32, S, kst, zk, zv, one, zero, o), Q.fp32_sq_norms(cfg32, S, nrm)),
        lambda m: (lambda out: Q.fp32_sq_norms(cfg32, S, out)))
    arms = {}
    runs = [(arm, 1) for arm in w.arms]
    if args.recall_lrb > 1:
        runs += [(arm, args.recall_lrb) for arm in w.arms if arm.policy != "yoked"]
    for arm, R in runs:
        cfg = Q.Config(T, dk, dv, arm.bits, arm.group, w.delta, w.decay, arm.policy, arm.rounding)
        st = Q.QState(cfg).init(torch.from_numpy(S0).to(dev))
        name = arm.name if R == 1 else f"{arm.name}+lrb{R}"
        if R == 1:
            stepf = (lambda i, want, st=st: st.step(kst, pool[1][i % P], pool[2][i % P],
                                                     pool[3][i % P], pool[4][i % P],
                                                     o if want else None))
            norms_at = lambda m, st=st, cfg=cfg: (lambda out: Q.state_sq_norms(cfg, st.codes, st.scales, out))
        else:
            buf = Q.LrbBuffers(cfg, R)
            stepf = (lambda i, want, st=st, buf=buf: buf.step(st, kst, pool[1][i % P], pool[2][i % P],
                                                               pool[3][i % P], pool[4][i % P],
                                                               o if want else None))
            norms_at = (lambda m, st=st, cfg=cfg, R=R:
                        (lambda out: Q.state_sq_norms(cfg, st.codes, st.scales, out)) if m % R == 0 else None)
        arms[name] = trajectory(
            stepf,
            lambda st=st, cfg=cfg: (st.readout(kst, o), Q.state_sq_norms(cfg, st.codes, st.scales, nrm)),
            norms_at)
    elapsed = time.time() - t0

    vs = vstar.astype(np.float64)
    med = lambda a: [None if not np.isfinite(x) else round(float(x), 6) for x in np.median(a, axis=1)]
    rel = lambda r, ref: np.linalg.norm(r - ref, axis=-1) / np.linalg.norm(ref, axis=-1)
    out = {"experiment": "recall over the decode horizon", "workload": w.description,
           "tiles": T, "steps": H, "checkpoints": marks, "launches": launches,
           "seconds": round(elapsed, 2), "read": "each step's readout with q = k*",
           "fp32": {"recall_err_vs_vstar": med(rel(fp[0], vs[None])),
                    "state_norm": med(np.sqrt(fp[1]))},
           "arms": {}}
    for name, (r, n) in arms.items():
        e = np.median(rel(r, fp[0]), axis=1)
        bad = [m for m, x in zip(marks, e) if x > args.recall_tol]
        out["arms"][name] = {
            "recall_err_vs_fp32": [round(float(x), 6) for x in e],
            "recall_err_vs_vstar": med(rel(r, vs[None])),
            "norm_ratio_vs_fp32": med(np.sqrt(n / fp[1])),
            "horizon": bad[0] if bad else None}
    out["horizon_rule"] = (f"first checkpoint where the median over tiles of "
                           f"||S_t k* - S_t^fp32 k*|| / ||S_t^fp32 k*|| exceeds {args.recall_tol}")
    print(json.dumps(out))


def prefill_flops(dk: int, dv: int, L: int, C: int = 32, delta: int = 0) -> int:
    """Algorithmic FLOPs of the chunkwise prefill of one tile over L tokens:
    per chunk of c tokens, the state read 2 c dk dv, the local scores c^2 dk
    (the causal half of 2 c^2 dk), the intra-chunk outputs c^2 dv and the
    state pass 2 c dk dv + dk dv; the delta rule adds the projection of the
    keys on the state 2 c dk dv, their scores c^2 dk and the forward
    substitution c^2 dv."""
    f = 0
    for c0 in range(0, L, C):
        c = min(C, L - c0)
        f += 4 * c * dk * dv + c * c * (dk + dv) + dk * dv
        if delta:
            f += 2 * c * dk * dv + c * c * (dk + dv)
    return f


def prefill_bytes(dk: int, dv: int, L: int, diag: bool) -> int:
    """Algorithmic HBM bytes of the prefill of one tile: q, k, v, alpha,
    beta read, o written, the FP32 state read and written."""
    return 4 * (L * (2 * dk + dv) + L * (dk if diag else 1) + L + L * dv + 2 * dv * dk)


def run_prefill(args):
    """Time the prefill paths over `--prefill` tokens for every tile of the
    workload (inputs drawn from its laws, slot t mod P for token t), from a
    zero state, with outputs (delta-rule workloads: the FP32 path only): qstate_prefill (FP32 on the CUDA cores, against
    the FP32 FMA peak of 148 SMs x 128 lanes x 2 FLOPs x the sampled SM
    clock) and qstate_prefill_tf32 (tensor cores, against the measured HBM
    copy bandwidth: its algorithmic bytes per launch / launch time, and its
    contraction FLOPs against the TF32 tensor peak, taken as half the
    measured bf16 peak, the nominal dense ratio).  Prints one JSON line."""
    import torch
    from ssm_decode_step_b200 import Config, qstate as Q
    w = W.get(args.workload)
    if args.prefill_tiles > 0:
        w = W.scaled_down(w, args.prefill_tiles, layers=1)
    L, P = args.prefill, max(1, min(args.pool or 64, args.prefill))
    dev = torch.device("cuda")
    T = w.tiles
    slots = [W.slot(w, t) for t in range(P)]
    idx = np.arange(L) % P
    arrs = [np.ascontiguousarray(np.stack([s[i] for s in slots], axis=1)[:, idx]) for i in range(5)]
    q, k, v, a, b = (torch.from_numpy(x).to(dev) for x in arrs)
    cfg = Config(T, w.dk, w.dv, 8, 32, w.delta, w.decay)
    S = torch.zeros((T, w.dv, w.dk), dtype=torch.float32, device=dev)
    o = torch.empty((T, L, w.dv), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    hbm_peak, hbm_src = load_peak()
    try:
        with open(PEAKS_FILE) as f:
            tf32_peak, tf32_src = 0.5 * float(json.load(f)["bf16_tflops"]), "measured bf16 x 0.5"
    except Exception:
        tf32_peak, tf32_src = 0.5 * 1590.0, "fallback bf16 x 0.5"
    out = {"experiment": "chunkwise prefill", "workload": w.description, "tiles": T,
           "tokens_per_tile": L, "launches": args.steps,
           "note": "the zeroing of S before every launch is inside the timed region (one memset)"}
    before = Q.prefill_tf32_timeouts()
    paths = [("fp32", Q.prefill)]
    if w.delta == 0:
        # timeouts are counted over the whole run below, not per call
        paths.append(("tf32", lambda *a: Q.prefill_tf32(*a, check_timeouts=False)))
    else:
        out["tf32"] = "not run: the tensor-core form covers the linear write (delta = 0) only"
    for name, fn in paths:
        for _ in range(args.warmup):
            fn(cfg, L, S, q, k, v, a, b, o)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(torch.cuda.current_device()) as sampler:
            e0.record(stream)
            for _ in range(args.steps):
                S.zero_()
                fn(cfg, L, S, q, k, v, a, b, o)
            e1.record(stream)
            torch.cuda.synchronize()
        clocks = sampler.summary()
        sec = e0.elapsed_time(e1) / 1e3 / args.steps
        mhz = clocks.get("sm_mhz") or 1965
        if name == "fp32":
            flops = T * prefill_flops(w.dk, w.dv, L, delta=w.delta)
            peak = 148 * 128 * 2 * mhz * 1e6 / 1e12
            out[name] = {"kernel": "prefill_kernel (CUDA cores, FP32)", "ms_per_prefill": round(sec * 1e3, 4),
                         "tokens_per_s": round(T * L / sec, 1), "tflops": round(flops / sec / 1e12, 3),
                         "fp32_peak_tflops": round(peak, 2),
                         "frac_of_fp32_peak": round(flops / sec / 1e12 / peak, 4), "bound": "alu",
                         "flops": "prefill_flops (chunks of 32)", "clocks": clocks}
        else:
            flops = T * prefill_flops(w.dk, w.dv, L, C=64)
            nbytes = T * prefill_bytes(w.dk, w.dv, L, w.decay == "diagonal")
            gbs = nbytes / sec / 1e9
            out[name] = {"kernel": "prefill_tc_kernel (tcgen05 TF32, accumulators in tensor memory)",
                         "ms_per_prefill": round(sec * 1e3, 4), "tokens_per_s": round(T * L / sec, 1),
                         "bytes_per_launch": nbytes, "gbs": round(gbs, 1), "hbm_peak_gbs": hbm_peak,
                         "hbm_peak_source": hbm_src, "frac_of_hbm_peak": round(gbs / hbm_peak, 4),
                         "bound": "hbm", "tflops": round(flops / sec / 1e12, 3),
                         "tf32_peak_tflops": round(tf32_peak, 1), "tf32_peak_source": tf32_src,
                         "frac_of_tf32_peak": round(flops / sec / 1e12 / tf32_peak, 4),
                         "flops": "prefill_flops (chunks of 64)", "clocks": clocks,
                         "speedup_vs_fp32": round(out["fp32"]["ms_per_prefill"] / (sec * 1e3), 2)}
    if w.delta == 0:
        out["tf32"]["timeouts"] = Q.prefill_tf32_timeouts() - before
    print(json.dumps(out))


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2048,
                    help="timed steps per arm")
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="stack24", choices=list(W.WORKLOADS))
    ap.add_argument("--pool", type=int, default=0,
                    help="input slots on the device (0: enough to exceed 2x L2, 16 to 64)")
    ap.add_argument("--groups", type=int, default=0, help="request groups (0: enough to exceed 2x L2)")
    ap.add_argument("--e2e-steps", type=int, default=1024)
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work")
    ap.add_argument("--ref-budget", type=float, default=90.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-fp32", action="store_true", help="skip the FP32-state comparison arm")
    ap.add_argument("--lrb-rank", type=int, default=8,
                    help="also time every arm with Low-Rank Bypass of this rank (0: skip)")
    ap.add_argument("--prefill", type=int, default=0,
                    help="time the chunkwise prefill over this many tokens per tile instead")
    ap.add_argument("--prefill-tiles", type=int, default=0,
                    help="with --prefill: that many tiles of the workload's laws (0: all)")
    ap.add_argument("--recall", action="store_true",
                    help="measure recall of a planted association over the decode horizon instead")
    ap.add_argument("--recall-steps", type=int, default=32768)
    ap.add_argument("--recall-tol", type=float, default=0.5)
    ap.add_argument("--recall-lrb", type=int, default=8,
                    help="also run the non-yoked arms with Low-Rank Bypass of this rank (0: skip)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.recall:
        run_recall(args)
    elif args.prefill > 0:
        run_prefill(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
