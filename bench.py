#!/usr/bin/env python
"""Benchmark of the selective-scan forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--quick]

One step is one call of ``ssm_scan_fwd`` on the Mamba-130M-layer-shaped
workload (batch 8, 1536 channels, 16 states, 2048 steps, bf16 u/delta/z/B/C,
fp32 A/D/bias, z gate on), inputs resident in HBM.  Rank 0 prints one JSON
line; ``value`` is the algorithmic HBM throughput (bytes every input read
once and every output written once, over the device time) summed over all
ranks.  Under torchrun every rank runs its own copy of the workload (the scan
has no exchange step: channels are independent), the timing is the maximum
over ranks, and scaling is weak.

Also reported: B*D*L elements/s, the fraction of the measured HBM copy
bandwidth, the ALU roofline of the dominant kernel (the scan at 16 states is
bound by its exponentials and fp32 lane operations, not by HBM), the same
metric end to end through the C ABI from pinned host buffers, clocks sampled
during the timed region, the CPU oracle as a baseline, and (without --quick)
one line per other workload: tiny fp32, the 2.8B-layer shape with and
without gate, the 2^20-step sequence, the scan with the convolution stage
fused in front, the scan's gradients, the Mamba-2 chunked scan, and the
decode step, eager and replayed from a CUDA graph.

``--impl reference`` times the CPU oracle instead, on a bounded sample of the
same workload per step, with the same metric and unit.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "mamba130m_layer"
METRIC = "selective_scan_fwd HBM GB/s (% of B200 peak) and B·D·L elems/s"
L2_FLUSH_BYTES = 512 << 20   # written between timed steps (L2 is 126 MB)
SM_COUNT_NOMINAL = 148
SM_MAX_MHZ_NOMINAL = 1965.0
FP32_LANES_PER_SM = 128      # measured on B200: 127.9 lane-ops/SM/clk
MUFU_LANES_PER_SM = 16       # measured: 16.0 ex2 / lg2 / tanh per SM per clk
EXP_POLY_LANE_OPS = 8        # FMA-pipe cost of one range-reduced degree-5 exp2


SCAN_SOURCES = ["scan_fwd.cuh", "common.cuh", "exp2_poly.cuh"]


def captured_traffic():
    """DRAM bytes per launch of the scan kernel from the recorded ncu capture,
    or None when the kernel sources changed since that capture."""
    import hashlib
    rec = {}
    try:
        with open(os.path.join(ROOT, "profiles", "scan_fwd_traffic.txt")) as f:
            for line in f:
                if line.strip() and not line.startswith("#"):
                    k, v = line.split()
                    rec[k] = v
        h = hashlib.sha256()
        for name in SCAN_SOURCES:
            with open(os.path.join(ROOT, "selective_state_space_08_b200", "csrc", name), "rb") as f:
                h.update(f.read())
    except (OSError, ValueError):
        return None
    if rec.get("sources_sha256") != h.hexdigest():
        return None
    return int(rec["dram_bytes_per_launch"])


def bf16_peak_tflops():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"])
    except (OSError, KeyError, ValueError):
        return 1590.0


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d.get("sm_max_mhz", SM_MAX_MHZ_NOMINAL)), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, SM_MAX_MHZ_NOMINAL, "fallback"


# ---------------------------------------------------------------------------- models
def scan_bytes(batch, dim, dstate, seqlen, esize, gate=True, h_last=True):
    """Algorithmic HBM bytes of one scan: each input read once, each output once."""
    x = batch * dim * seqlen * esize
    total = x * (2 + (1 if gate else 0))      # u, delta (, z)
    total += x                                 # y
    total += 2 * batch * dstate * seqlen * esize  # B, C
    total += dim * dstate * 4 + 2 * dim * 4    # A, D, bias
    if h_last:
        total += batch * dim * dstate * 4
    return total


def ssd_bytes(batch, seqlen, nheads, headdim, dstate, gate=False, h0=False):
    """Algorithmic HBM bytes of one chunked scan (bf16 tensors, fp32 state)."""
    x = batch * seqlen * nheads * headdim * 2
    total = 2 * x + (x if gate else 0)               # x, y (, z)
    total += 2 * batch * seqlen * dstate * 2          # B, C
    total += batch * seqlen * nheads * 2              # delta
    total += batch * nheads * headdim * dstate * 4 * (2 if h0 else 1)  # h_last (, h0)
    total += 3 * nheads * 4
    return total


def ssd_flops(batch, seqlen, nheads, headdim, dstate, chunk):
    """Dense tensor-core FLOPs of the chunked form: C B^T per (batch, chunk),
    and per head the masked Q x Q product with X', the chunk state and the
    read-out of the carried state."""
    nc = -(-seqlen // chunk)
    g = 2 * chunk * chunk * dstate
    per_head = 2 * chunk * chunk * headdim + 2 * 2 * chunk * dstate * headdim
    return batch * nc * (g + nheads * per_head)


def alu_cycles_per_elem(dstate, gate=True, softplus=True):
    """SM cycles per (b, d, t) element at the FP32/MUFU limit.

    Per element the method needs dstate exponentials exp(dt' A) plus, per
    element, softplus (an exp and a log) and the gate (an exp and a
    reciprocal): transcendentals n_tr.  FP32 lane-operations: 4 per state
    (dt' A, dt' u B, the state FMA, the C.h FMA) plus 4 per element.  A
    transcendental costs 1 of the 16 MUFU lanes, or EXP_POLY_LANE_OPS of the
    128 FP32 lanes when evaluated as a polynomial; the split s that balances
    the two pipes gives the bound."""
    n_tr = dstate + (2 if softplus else 0) + (2 if gate else 0)
    n_fma = 4 * dstate + 4
    c = EXP_POLY_LANE_OPS
    ratio = FP32_LANES_PER_SM / MUFU_LANES_PER_SM
    s = min(1.0, (n_fma + n_tr * c) / (n_tr * (ratio + c)))
    return max(s * n_tr / MUFU_LANES_PER_SM, (n_fma + (1 - s) * n_tr * c) / FP32_LANES_PER_SM)


def alu_peak_elems(dstate, gate=True, sms=SM_COUNT_NOMINAL, mhz=SM_MAX_MHZ_NOMINAL):
    return sms * mhz * 1e6 / alu_cycles_per_elem(dstate, gate)


# ---------------------------------------------------------------------------- clocks
class ClockSampler:
    """Polls the SM clock and the clock-event reasons through NVML (what
    nvidia-smi reports) every 2 ms while running."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index):
        self.samples, self.reasons, self.max_mhz = [], 0, None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = self._handle(pynvml, index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:  # noqa: BLE001 -- no NVML: no clock record
            self._nv = None
        self._t = threading.Thread(target=self._run, daemon=True)

    @staticmethod
    def _handle(nv, index):
        """NVML handle of CUDA device ``index``, matched by UUID: the CUDA and
        NVML numberings differ when CUDA_VISIBLE_DEVICES remaps devices."""
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(index).uuid)
            return nv.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:  # noqa: BLE001 -- fall back to the same index
            return nv.nvmlDeviceGetHandleByIndex(index)

    def _sample(self):
        nv = self._nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
        try:
            r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
        except Exception:  # noqa: BLE001
            r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self._h)
        self.reasons |= int(r)

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(0.002)

    def __enter__(self):
        if self._nv is not None:
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self._nv is not None:
            self._stop.set()
            self._t.join()
            self._sample()

    def record(self):
        if self._nv is None or not self.samples:
            return None
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "samples": len(self.samples), "reasons": names}


# ---------------------------------------------------------------------------- helpers
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def reduce_max(value: float, world: int, device=None) -> float:
    """Maximum of ``value`` over all ranks (identity on one rank)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_value(units_per_rank: float, world: int, seconds_max: float) -> float:
    """Whole-job throughput: every rank's units over the slowest rank's time."""
    return units_per_rank * world / seconds_max


def workload_cfg(name):
    from selective_state_space_08_b200 import synth
    return dict(synth.CONFIGS[name])


def describe(cfg, gate):
    return (f"batch={cfg['batch']} dim={cfg['dim']} dstate={cfg['dstate']} "
            f"seqlen={cfg['seqlen']} {cfg['dtype']} gate={'on' if gate else 'off'}")


# ---------------------------------------------------------------------------- our arm
class ScanCase:
    """Device-resident inputs and outputs of one selective-scan workload."""

    def __init__(self, name, gate=None, device="cuda"):
        import numpy as np
        import torch
        from selective_state_space_08_b200 import synth
        cfg = workload_cfg(name)
        if gate is not None:
            cfg["gate"] = gate
        self.cfg, self.name = cfg, name
        host = synth.make_scan_inputs(cfg["batch"], cfg["dim"], cfg["dstate"], cfg["seqlen"],
                                      cfg["dtype"], cfg["gate"], cfg["seed"], cfg["s_range"],
                                      bits=True)
        self.host = host
        tdt = torch.bfloat16 if cfg["dtype"] == "bf16" else torch.float32

        def up(a):
            if a is None:
                return None
            if a.dtype == np.uint16:
                return torch.from_numpy(a.view(np.int16)).to(device).view(torch.bfloat16)
            return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)

        self.t = {k: up(v) for k, v in host.items()}
        self.esize = 2 if tdt == torch.bfloat16 else 4
        self.y = torch.empty(self.t["u"].shape, dtype=tdt, device=device)
        self.h = torch.empty((cfg["batch"], cfg["dim"], cfg["dstate"]), dtype=torch.float32,
                             device=device)
        self.ws = None
        from selective_state_space_08_b200 import api
        need = api.scan_fwd_workspace_size(*self.args()[:5])
        self.launches = 3 if need > 0 else 1
        if need:
            self.ws = torch.empty(need, dtype=torch.uint8, device=device)
        self.bytes = scan_bytes(cfg["batch"], cfg["dim"], cfg["dstate"], cfg["seqlen"], self.esize,
                                cfg["gate"])
        self.elems = cfg["batch"] * cfg["dim"] * cfg["seqlen"]

    def args(self):
        t = self.t
        return [t["u"], t["delta"], t["A"], t["B"], t["C"], t["D"], t["z"], t["delta_bias"], True,
                None]

    def step(self):
        from selective_state_space_08_b200 import api
        api.scan_fwd(*self.args(), y=self.y, h_last=self.h, workspace=self.ws)


class nvtx_range:
    """An NVTX range around a block (visible to Nsight tools, e.g. ncu's
    --nvtx-include); does nothing where NVTX is unavailable."""

    def __init__(self, name):
        self.name, self.on = name, False

    def __enter__(self):
        try:
            import torch
            torch.cuda.nvtx.range_push(self.name)
            self.on = True
        except Exception:  # noqa: BLE001 -- profiling aid only
            pass
        return self

    def __exit__(self, *exc):
        if self.on:
            try:
                import torch
                torch.cuda.nvtx.range_pop()
            except Exception:  # noqa: BLE001
                pass


def time_steps(step, steps, warmup, flush, world, device, sampler_index=None, name="steps"):
    """W untimed steps, then K steps each bracketed by CUDA events on the
    launching stream, with an L2 flush (outside the events) between them.
    Returns (sum of step times in seconds, max over ranks; per-step ms; clocks)."""
    import torch
    import torch.distributed as dist
    with nvtx_range(f"{name}: warm-up"):
        for _ in range(warmup):
            step()
        torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(sampler_index if sampler_index is not None else 0)
    with sampler, nvtx_range(f"{name}: timed"):
        for k in range(steps):
            flush.zero_()
            starts[k].record()
            step()
            ends[k].record()
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    per = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total = reduce_max(sum(per) / 1e3, world, device)
    return total, per, sampler.record()


def e2e_measure(case, steps, warmup, slice_batch=2):
    """The same metric through the C ABI from page-locked host buffers
    (ssm_scan_fwd_host): per step the host->device copies of every input, the
    scan and the device->host copies of y and h_last, all inside the timed
    region.  The call pipelines batch slices of ``slice_batch`` sequences, so
    the copies in both directions overlap each other and the scans."""
    import numpy as np
    import torch
    from selective_state_space_08_b200 import api
    names = ["u", "delta", "A", "B", "C", "D", "z", "delta_bias"]
    pinned = {k: case.t[k].cpu().pin_memory() for k in names if case.t[k] is not None}
    y_host = torch.empty(case.y.shape, dtype=case.y.dtype).pin_memory()
    h_host = torch.empty(case.h.shape, dtype=torch.float32).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in pinned.values())
    d2h = y_host.numel() * y_host.element_size() + h_host.numel() * 4
    args = [pinned["u"], pinned["delta"], pinned["A"], pinned["B"], pinned["C"], pinned.get("D"),
            pinned.get("z"), pinned.get("delta_bias"), True, None]
    staging = torch.empty(api.scan_fwd_host_staging_size(*args, slice_batch=slice_batch),
                          dtype=torch.uint8, device="cuda")

    def one():
        api.scan_fwd_host(*args, y=y_host, h_last=h_host, slice_batch=slice_batch,
                          staging=staging, synchronize=False)

    for _ in range(warmup):
        one()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(steps):
        one()
    e.record()
    torch.cuda.synchronize()
    sec = s.elapsed_time(e) / 1e3 / steps
    assert bool(np.isfinite(y_host.float().numpy()).all())
    return {"value": round(case.bytes / sec / 1e9, 2), "unit": "GB/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "ms_per_step": round(sec * 1e3, 4), "api": "ssm_scan_fwd_host",
            "slice_batch": slice_batch}


def oracle_baseline(case_host, cfg, gate, batches):
    """The CPU oracle as it stands on the host cores, on ``batches`` of the workload."""
    import numpy as np
    import oracle
    from selective_state_space_08_b200 import synth
    cores = os.cpu_count() or 1

    def f(a, b):
        if a is None:
            return None
        v = a[b] if a.ndim == 3 else a
        return synth.bf16_bits_to_f32(v).reshape(v.shape) if v.dtype == np.uint16 else v

    t0 = time.perf_counter()
    for b in batches:
        oracle.scan_fwd(f(case_host["u"], b)[None], f(case_host["delta"], b)[None], case_host["A"],
                        f(case_host["B"], b)[None], f(case_host["C"], b)[None], case_host["D"],
                        f(case_host["z"], b)[None] if gate else None, case_host["delta_bias"],
                        True, None, nthreads=cores)
    sec = time.perf_counter() - t0
    nb = len(batches)
    bytes_ = scan_bytes(nb, cfg["dim"], cfg["dstate"], cfg["seqlen"],
                        2 if cfg["dtype"] == "bf16" else 4, gate)
    elems = nb * cfg["dim"] * cfg["seqlen"]
    return {"value": round(bytes_ / sec / 1e9, 4), "unit": "GB/s", "cores": cores,
            "kind": "oracle", "elems_per_s": round(elems / sec, 1), "seconds": round(sec, 3),
            "sample": (f"{nb} of {cfg['batch']} batches of the {WORKLOAD} workload "
                       f"({elems} elements), float64, {cores} threads")}


def ssd_case():
    """Device-resident inputs of the Mamba-2 layer workload and the call that
    runs the chunked scan on them: (config, call, tensors to keep alive)."""
    import torch
    from selective_state_space_08_b200 import api, synth
    cfg = workload_cfg("mamba2_ssd")
    sin = synth.make_ssd_inputs(cfg["batch"], cfg["seqlen"], cfg["nheads"], cfg["headdim"],
                                cfg["dstate"], cfg["dtype"], cfg["gate"], cfg["seed"], cfg["s_range"])
    bfd = lambda a: torch.from_numpy(a).cuda().to(torch.bfloat16)
    f32d = lambda a: torch.from_numpy(a).cuda()
    sx, sdl, sB, sC = bfd(sin["x"]), bfd(sin["delta"]), bfd(sin["B"]), bfd(sin["C"])
    sA, sD, sbias = f32d(sin["A"]), f32d(sin["D"]), f32d(sin["delta_bias"])
    sy = torch.empty_like(sx)
    sh = torch.empty((cfg["batch"], cfg["nheads"], cfg["headdim"], cfg["dstate"]),
                     dtype=torch.float32, device="cuda")
    sws = torch.empty(api.ssd_workspace_size(cfg["batch"], cfg["seqlen"], cfg["nheads"],
                                             cfg["headdim"], cfg["dstate"], cfg["chunk"]),
                      dtype=torch.uint8, device="cuda")
    sstep = lambda: api.ssd_fwd(sx, sdl, sA, sB, sC, sD, None, sbias, True, None,
                                chunk=cfg["chunk"], y=sy, h_last=sh, workspace=sws)
    return cfg, sstep, (sx, sdl, sB, sC, sA, sD, sbias, sy, sh, sws)


def run_profile(args):
    """Runs only the product call of one workload, warmup + steps times, with
    no timing, flush or output line: the command an ncu capture wraps
    (select the launch with ncu's -k / -s / -c)."""
    import torch
    torch.cuda.set_device(0)
    if args.profile == "scan":
        case = ScanCase(WORKLOAD)
        step = case.step
    elif args.profile == "bwd":
        from selective_state_space_08_b200 import api
        case = ScanCase(WORKLOAD)
        t = case.t
        dy = torch.randn(t["u"].shape, dtype=torch.float32, device="cuda")
        bws = torch.empty(api.scan_bwd_workspace_size(t["u"], t["delta"], t["A"], t["B"], t["C"],
                                                      t["D"], t["z"], t["delta_bias"], True),
                          dtype=torch.uint8, device="cuda")
        step = lambda: api.scan_bwd(t["u"], t["delta"], t["A"], t["B"], t["C"], dy, t["D"],
                                    t["z"], t["delta_bias"], True, None, workspace=bws)
    else:
        _, step, keep = ssd_case()
    for _ in range(args.warmup + args.steps):
        step()
    torch.cuda.synchronize()
    print(f"profile: {args.warmup + args.steps} calls of the {args.profile} workload")


def extra_workloads(steps, warmup, flush, hbm_peak):
    import torch
    from selective_state_space_08_b200 import api, synth
    out = {}
    for name, gate in (("tiny_fp32", True), ("mamba2p8b_layer", True), ("mamba2p8b_layer", False),
                       ("long_seq", True)):
        case = ScanCase(name, gate)
        reps = steps if name != "long_seq" else max(3, min(steps, 10))
        total, per, _ = time_steps(case.step, reps, min(warmup, 3), flush, 1, None, name=name)
        sec = total / reps
        key = f"{name}{'' if gate else '_nogate'}"
        out[key] = {"config": describe(case.cfg, gate), "us_per_call": round(sec * 1e6, 2),
                    "GB_per_s": round(case.bytes / sec / 1e9, 1),
                    "hbm_frac": round(case.bytes / sec / 1e9 / hbm_peak, 4),
                    "elems_per_s": round(case.elems / sec, 1),
                    "alu_frac": round(case.elems / sec / alu_peak_elems(case.cfg["dstate"], gate), 4),
                    "launches_per_call": case.launches}
        del case
        torch.cuda.empty_cache()
    # the scan with the convolution stage fused in front (width 4), 130M-layer shape
    case = ScanCase(WORKLOAD)
    conv = synth.make_conv_params(case.cfg["dim"], 4, seed=1)
    cw = torch.from_numpy(conv["weight"]).cuda()
    cb = torch.from_numpy(conv["bias"]).cuda()
    t = case.t
    cstep = lambda: api.scan_fwd_conv(t["u"], cw, cb, None, t["delta"], t["A"], t["B"], t["C"],
                                      t["D"], t["z"], t["delta_bias"], True, None, y=case.y,
                                      h_last=case.h, workspace=case.ws)
    total, per, _ = time_steps(cstep, steps, warmup, flush, 1, None, name="conv stage")
    sec = total / steps
    cbytes = case.bytes + cw.numel() * 4 + cb.numel() * 4
    out["mamba130m_layer_conv"] = {
        "config": describe(case.cfg, True) + ", conv width 4 fused in front",
        "us_per_call": round(sec * 1e6, 2), "GB_per_s": round(cbytes / sec / 1e9, 1),
        "hbm_frac": round(cbytes / sec / 1e9 / hbm_peak, 4),
        "elems_per_s": round(case.elems / sec, 1),
        "alu_frac": round(case.elems / sec / alu_peak_elems(case.cfg["dstate"], True), 4),
        "launches_per_call": case.launches}
    del case, cstep
    torch.cuda.empty_cache()
    # gradients of the scan on the 130M-layer shape (dy fp32, gradients fp32)
    case = ScanCase(WORKLOAD)
    t = case.t
    dy = torch.randn(t["u"].shape, dtype=torch.float32, device="cuda")
    bws = torch.empty(api.scan_bwd_workspace_size(t["u"], t["delta"], t["A"], t["B"], t["C"],
                                                  t["D"], t["z"], t["delta_bias"], True),
                      dtype=torch.uint8, device="cuda")
    bstep = lambda: api.scan_bwd(t["u"], t["delta"], t["A"], t["B"], t["C"], dy, t["D"], t["z"],
                                 t["delta_bias"], True, None, workspace=bws)
    total, per, _ = time_steps(bstep, max(3, steps // 4), warmup, flush, 1, None, name="gradients")
    sec = total / max(3, steps // 4)
    c = case.cfg
    elems = c["batch"] * c["dim"] * c["seqlen"]
    bc = 2 * c["batch"] * c["dstate"] * c["seqlen"]
    bbytes = elems * (3 * case.esize + 4 + 3 * 4) + bc * (case.esize + 4)
    out["mamba130m_layer_bwd"] = {
        "config": describe(c, True) + ", gradients of every input (fp32)",
        "us_per_call": round(sec * 1e6, 2), "GB_per_s": round(bbytes / sec / 1e9, 1),
        "hbm_frac": round(bbytes / sec / 1e9 / hbm_peak, 4),
        "elems_per_s": round(elems / sec, 1), "launches_per_call": 2}
    del case, dy, bws, bstep
    torch.cuda.empty_cache()
    # Mamba-2 chunked scan (tensor cores)
    cfg, sstep, keep = ssd_case()
    total, per, _ = time_steps(sstep, steps, warmup, flush, 1, None, name="chunked scan")
    sec = total / steps
    sb = ssd_bytes(cfg["batch"], cfg["seqlen"], cfg["nheads"], cfg["headdim"], cfg["dstate"])
    sf = ssd_flops(cfg["batch"], cfg["seqlen"], cfg["nheads"], cfg["headdim"], cfg["dstate"],
                   cfg["chunk"])
    out["mamba2_ssd"] = {
        "config": (f"batch={cfg['batch']} seqlen={cfg['seqlen']} nheads={cfg['nheads']} "
                   f"headdim={cfg['headdim']} dstate={cfg['dstate']} chunk={cfg['chunk']} bf16"),
        "us_per_call": round(sec * 1e6, 2), "GB_per_s": round(sb / sec / 1e9, 1),
        "hbm_frac": round(sb / sec / 1e9 / hbm_peak, 4),
        "TFLOP_per_s": round(sf / sec / 1e12, 1),
        "tensor_frac_of_measured_bf16": round(sf / sec / 1e12 / bf16_peak_tflops(), 4),
        "launches_per_call": 3}
    del sstep, keep
    torch.cuda.empty_cache()
    # decode step on the 2.8B-layer channel count (batch 4 x 5120 channels)
    cfg = workload_cfg("mamba2p8b_layer")
    B_, D_, N_ = cfg["batch"], cfg["dim"], cfg["dstate"]
    inp = synth.make_scan_inputs(B_, D_, N_, 1, "bf16", True, 7, h0=True)
    dev = lambda a, bf=True: (torch.from_numpy(a).cuda().to(torch.bfloat16) if bf
                              else torch.from_numpy(a).cuda())
    st = dev(inp["h0"], False).contiguous()
    args = [dev(inp["u"][..., 0].copy()), dev(inp["delta"][..., 0].copy()), dev(inp["A"], False),
            dev(inp["B"][..., 0].copy()), dev(inp["C"][..., 0].copy()), dev(inp["D"], False),
            dev(inp["z"][..., 0].copy()), dev(inp["delta_bias"], False)]
    yv = torch.empty((B_, D_), dtype=torch.bfloat16, device="cuda")
    step = lambda: api.scan_step(st, *args, y=yv)
    total, per, _ = time_steps(step, steps, warmup, flush, 1, None, name="decode step")
    sec = total / steps
    sbytes = B_ * D_ * N_ * 8 + B_ * D_ * 2 * 4 + 2 * B_ * N_ * 2 + D_ * (N_ + 2) * 4
    out["decode_step"] = {"config": f"batch={B_} dim={D_} dstate={N_} bf16 gate=on, state fp32",
                          "us_per_call": round(sec * 1e6, 3),
                          "GB_per_s": round(sbytes / sec / 1e9, 1),
                          "hbm_frac": round(sbytes / sec / 1e9 / hbm_peak, 4)}
    # the same step, 64 steps per CUDA-graph replay (no per-call launch latency)
    T = 64
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(T):
            step()
    total, per, _ = time_steps(graph.replay, max(3, steps // 8), warmup, flush, 1, None,
                               name="decode graph")
    sec = total / max(3, steps // 8) / T
    out["decode_step_graph"] = {"config": f"{out['decode_step']['config']}, {T} steps per graph replay",
                                "us_per_call": round(sec * 1e6, 3),
                                "GB_per_s": round(sbytes / sec / 1e9, 1),
                                "hbm_frac": round(sbytes / sec / 1e9 / hbm_peak, 4)}
    del graph
    return out


def run_ours(args):
    import torch
    import torch.distributed as dist
    world, rank, local = dist_env()
    torch.cuda.set_device(local)  # before the process group, so NCCL binds this rank's GPU
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    device = torch.device("cuda", local)
    hbm_peak, sm_max_mhz, peak_kind = peaks()
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)

    case = ScanCase(WORKLOAD, device=device)
    total, per, clocks = time_steps(case.step, args.steps, args.warmup, flush, world, device,
                                    sampler_index=local, name=WORKLOAD)
    sec = total / args.steps
    value = weak_value(case.bytes, world, sec) / 1e9
    elems_s = weak_value(case.elems, world, sec)
    kernel_s = statistics.mean(per) / 1e3  # one kernel launch per step on this workload
    alu_peak = alu_peak_elems(case.cfg["dstate"], case.cfg["gate"], mhz=sm_max_mhz)
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(sec * 1e3, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) inputs, log-uniform decays and steps)",
        "config": {"workload": f"{WORKLOAD}: {describe(case.cfg, case.cfg['gate'])}",
                   "elements_per_step_per_gpu": case.elems,
                   "algorithmic_bytes_per_step_per_gpu": case.bytes,
                   "l2": f"flushed between timed steps ({L2_FLUSH_BYTES >> 20} MiB write)",
                   "parallelism": f"replicas x{world} (independent channels, no exchange)"},
        "elems_per_s": round(elems_s, 1),
        "hbm_frac": round(value / world / hbm_peak, 4),
        "hbm_peak_gbs": hbm_peak, "hbm_peak_kind": peak_kind,
        "roofline": {"bound": "alu", "achieved": round(case.elems / kernel_s / 1e9, 2),
                     "peak": round(alu_peak / 1e9, 2), "unit": "Gelem/s",
                     "frac": round(case.elems / kernel_s / alu_peak, 4),
                     "traffic": captured_traffic(),
                     "traffic_unit": "bytes per launch (dram read + write, ncu)",
                     "kernel": "scan_fwd_kernel<bf16, full, gate>",
                     "hbm_achieved_gbs": round(case.bytes / kernel_s / 1e9, 1),
                     "hbm_frac": round(case.bytes / kernel_s / 1e9 / hbm_peak, 4),
                     "peak_derivation": (f"{SM_COUNT_NOMINAL} SMs x {sm_max_mhz:.0f} MHz / "
                                         f"{alu_cycles_per_elem(case.cfg['dstate'], case.cfg['gate']):.4f}"
                                         " SM-cycles per element (FP32 128 + MUFU 16 lanes/clk)")},
        "gpu_launches": case.launches * args.steps,
        "clocks": clocks,
    }
    if rank == 0 and world == 1:
        line["e2e"] = e2e_measure(case, max(3, min(args.steps, 20)), 2)
        line["cpu_baseline"] = oracle_baseline(case.host, case.cfg, case.cfg["gate"],
                                               list(range(case.cfg["batch"])))
        if not args.quick:
            del case
            torch.cuda.empty_cache()
            line["workloads"] = extra_workloads(min(args.steps, 20), max(args.warmup, 3), flush,
                                                hbm_peak)
    elif world > 1:
        # every rank moves its own replica's data at the same time (the host
        # links may be shared); the slowest rank's time sets the value
        dist.barrier()
        e2e = e2e_measure(case, max(3, min(args.steps, 20)), 2)
        sec = reduce_max(e2e["ms_per_step"] / 1e3, world, device)
        e2e["ms_per_step"] = round(sec * 1e3, 4)
        e2e["value"] = round(weak_value(case.bytes, world, sec) / 1e9, 2)
        e2e["note"] = "all ranks at once; max over ranks of the time per step"
        line["e2e"] = e2e
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# ---------------------------------------------------------------------------- reference arm
def run_reference(args):
    """The CPU oracle, timed as it stands on the host cores: each step one
    batch (1536 channels x 2048 steps) of the same workload."""
    world, rank, _ = dist_env()
    if rank != 0:
        return
    from selective_state_space_08_b200 import synth
    cfg = workload_cfg(WORKLOAD)
    host = synth.make_scan_inputs(1, cfg["dim"], cfg["dstate"], cfg["seqlen"], cfg["dtype"],
                                  cfg["gate"], cfg["seed"], cfg["s_range"], bits=True)
    for _ in range(args.warmup):
        oracle_baseline(host, cfg, cfg["gate"], [0])
    t0 = time.perf_counter()
    last = None
    for _ in range(args.steps):
        last = oracle_baseline(host, cfg, cfg["gate"], [0])
    sec = (time.perf_counter() - t0) / args.steps
    bytes_ = scan_bytes(1, cfg["dim"], cfg["dstate"], cfg["seqlen"], 2, cfg["gate"])
    value = bytes_ / sec / 1e9
    cores = os.cpu_count() or 1
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(sec * 1e3, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"{WORKLOAD}: {describe(cfg, cfg['gate'])}",
                       "sample_per_step": "batch 0 of 8 (1536 channels x 2048 steps)"},
            "elems_per_s": round(cfg["dim"] * cfg["seqlen"] / sec, 1),
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores,
                             "kind": "oracle", "sample": last["sample"]},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--quick", action="store_true", help="skip the other workloads")
    ap.add_argument("--profile", choices=["scan", "bwd", "ssd"], default=None,
                    help="only run the product call of the scan (mamba130m_layer), its\n"
                         "gradients (same shape) or the chunked-scan (mamba2_ssd)\n"
                         "workload warmup + steps times, untimed, for a profiler to capture")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.profile is not None:
        run_profile(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
