"""Benchmark of the selective scan forward (and the decode step) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

One step = one selective-scan forward (mamba_scan_fwd through the C ABI) over
the 130M-class layer: batch 8, d_inner 1536, d_state 16, L 2048, bf16 inputs,
fp32 y and last_state. Inputs are synthetic, seeded, resident in HBM; three
copies of them (and two of y) are rotated so that every step reads inputs not
touched by the two previous steps (254 MB per set, above the 126 MB L2). Rank
0 prints one JSON line. Under torchrun every rank runs its own layer (weak
scaling, no collective on the data path); the device time is the max over
ranks. The same line carries legs for the other forward workloads (2.8B-class
layer, long context), the decode step and the widened entry points, each with
its bytes, time, roofline fraction and clocks.

`--impl reference` times the fp64 CPU oracle on the host cores instead, on a
bounded sample of the same workload per step.
"""
from __future__ import annotations

import argparse
import hashlib
import glob
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "selective-scan fwd achieved HBM GB/s and Gchannel-tokens/s vs HBM roofline"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0


# ------------------------------------------------------------ byte models ----

def scan_bytes(batch, dim, dstate, seqlen, in_bytes, out_bytes):
    """Minimum HBM bytes of one scan: u, delta, z read and y written per
    channel-token; B, C read once per (batch, token); A read, D and bias read,
    last_state written."""
    ct = batch * dim * seqlen
    return (ct * (3 * in_bytes + out_bytes) + batch * seqlen * 2 * dstate * in_bytes
            + batch * dim * dstate * 4 + dim * dstate * 4 + 2 * dim * 4)


def decode_bytes(batch, dim, dstate, in_bytes, out_bytes):
    """Minimum HBM bytes of one decode step: the fp32 state read and written,
    x, delta, z read and y written per channel, B and C per batch row, A, D,
    bias."""
    return (batch * dim * dstate * 8 + batch * dim * (3 * in_bytes + out_bytes)
            + batch * dstate * 2 * in_bytes + dim * dstate * 4 + 2 * dim * 4)


def bwd_bytes(batch, dim, dstate, seqlen, in_bytes, out_bytes):
    """Minimum HBM bytes of one backward: u, delta, z and dout read and du,
    ddelta, dz (fp32) written per channel-token; B, C read and dB, dC (fp32)
    written per (batch, token); the saved states read; A, D, bias read and
    their gradients and dinitial_state written."""
    ct = batch * dim * seqlen
    nck = (seqlen + 63) // 64
    return (ct * (3 * in_bytes + out_bytes + 3 * 4) + batch * seqlen * 2 * dstate * (in_bytes + 4)
            + batch * dim * nck * dstate * 4 + batch * dim * dstate * 4 + 2 * (dim * dstate * 4 + 2 * dim * 4))


def ssd_bytes(batch, seqlen, nheads, headdim, dstate, ngroups, in_bytes, out_bytes):
    """Minimum HBM bytes of one SSD layer forward: x and dt read, y written,
    B and C read once per (batch, token, group), A/D/dt_bias read and the
    final state written."""
    return (batch * seqlen * nheads * (headdim * (in_bytes + out_bytes) + in_bytes)
            + batch * seqlen * ngroups * 2 * dstate * in_bytes + 3 * nheads * 4
            + batch * nheads * headdim * dstate * 4)


def ssd_flops(batch, seqlen, nheads, headdim, dstate, chunk=128):
    """Multiply-adds x 2 of the chunked matrix view per (batch, head, chunk):
    C S_in (Q N P), C B^T (Q Q N), G' X (Q Q P), B'^T X (N Q P)."""
    nch = (seqlen + chunk - 1) // chunk
    per = 2 * (chunk * dstate * headdim + chunk * chunk * dstate + chunk * chunk * headdim + dstate * chunk * headdim)
    return batch * nheads * nch * per


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def measured_bf16_tflops():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"])
    except Exception:
        return 1590.0


def ssd_bound(nbytes, flops, hbm_gbs, tflops):
    """Which roofline bounds the chunked SSD launch: its bytes at the HBM peak
    against its flops at the bf16 tensor peak, the slower one."""
    t_hbm = nbytes / (hbm_gbs * 1e9)
    t_tc = flops / (tflops * 1e12)
    which = "hbm" if t_hbm >= t_tc else "tensor"
    return f"{which} (bytes / {hbm_gbs:.0f} GB/s: {t_hbm * 1e3:.4f} ms; flops / {tflops:.0f} TFLOP/s: {t_tc * 1e3:.4f} ms)"


# B200 HBM3e nominal bandwidth (GB/s), printed beside the graded fraction of
# the measured copy peak
NOMINAL_HBM_GBS = 8000.0

# Sources that decide what a recorded kernel does: its own file, the shared
# device and argument headers, the public header and the ABI layer (which
# chooses the launch).
_SHARED_SOURCES = ("selective_state_space_40_b200/csrc/ms_device.cuh", "selective_state_space_40_b200/csrc/ms_internal.h",
                   "selective_state_space_40_b200/csrc/mambascan_api.cu", "include/mambascan.h")
KERNEL_SOURCES = {
    "scan_fwd_130m": ("selective_state_space_40_b200/csrc/scan_fwd.cu",
                      "selective_state_space_40_b200/csrc/scan_fwd_tmem.cu"),
    "scan_fwd_2p8b": ("selective_state_space_40_b200/csrc/scan_fwd.cu",
                      "selective_state_space_40_b200/csrc/scan_fwd_tmem.cu"),
    "scan_fwd_long": ("selective_state_space_40_b200/csrc/scan_fwd.cu",
                      "selective_state_space_40_b200/csrc/scan_fwd_tmem.cu"),
    "conv_scan_130m": ("selective_state_space_40_b200/csrc/scan_fwd.cu",
                       "selective_state_space_40_b200/csrc/scan_fwd_tmem.cu"),
    "decode_step": ("selective_state_space_40_b200/csrc/state_update_stream.cu",),
    "scan_bwd_130m": ("selective_state_space_40_b200/csrc/scan_bwd.cu",),
    "ssd_2p7b": ("selective_state_space_40_b200/csrc/ssd_fwd_tc.cu",),
    "ssd_decode": ("selective_state_space_40_b200/csrc/ssd_update.cu",),
}


def csrc_digest(kernel=None):
    """Hash of the sources of one recorded kernel (all of csrc/ when kernel is None)."""
    if kernel is None:
        paths = sorted(glob.glob(os.path.join(ROOT, "selective_state_space_40_b200", "csrc", "*")))
    else:
        paths = [os.path.join(ROOT, p) for p in sorted(KERNEL_SOURCES[kernel] + _SHARED_SOURCES)]
    h = hashlib.sha256()
    for p in paths:
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel):
    """DRAM bytes per launch from the committed ncu capture, if it was taken
    on the kernel's current sources (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(kernel)
    except Exception:
        return None
    if not rec or kernel not in KERNEL_SOURCES or rec.get("csrc_sha") != csrc_digest(kernel):
        return None
    return rec.get("dram_bytes_per_launch")


# ----------------------------------------------------------- clock sampler ----

class ClockSampler:
    """Samples the SM clock and the clock-event reasons through NVML while the
    timed region runs (reads only; changes no setting)."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, device_index, period=0.02):
        self.period = period
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception:
            self._ok = False

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
                r = self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for name, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._ok:
            self._t.join()

    def summary(self):
        if not self._ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["nvml unavailable"],
                    "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


# ------------------------------------------------------------- dist plumbing --

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world, backend):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        import datetime
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(value, world, device=None):
    """Max of a per-rank float over all ranks (identity for one rank)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# -------------------------------------------------------------- timing ----

def time_launches(torch, stream, fn, steps, warmup, device_index):
    """Mean per-launch time (ms) of fn(i) with CUDA events on the launching
    stream, after `warmup` untimed launches; the NVML clock record of the
    timed launches beside it."""
    for i in range(warmup):
        fn(i)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    torch.cuda.synchronize()
    with ClockSampler(device_index, period=0.001) as clk:
        for i in range(steps):
            ev[i][0].record(stream)
            fn(warmup + i)
            ev[i][1].record(stream)
        torch.cuda.synchronize()
    return statistics.fmean(a.elapsed_time(b) for a, b in ev), clk.summary()


def forward_leg(torch, mb, syn, w, stream, dev, local, world, peak, steps, nsets, traffic_key):
    """One forward workload timed launch by launch over `nsets` rotating input
    sets (each above the 126 MB L2), automatic plan, fp32 y and last_state."""
    es = 2 if w.in_dtype == torch.bfloat16 else 4
    host = syn.scan_inputs(w)
    sets = [{k: v.to(dev) for k, v in host.items()} for _ in range(nsets)]
    del host
    y = torch.empty(w.batch, w.dim, w.seqlen, dtype=torch.float32, device=dev)
    last = torch.empty(w.batch, w.dim, w.dstate, dtype=torch.float32, device=dev)
    dims = mb.scan_dims_for(sets[0]["u"], sets[0]["delta"], sets[0]["B"], sets[0]["C"], sets[0]["z"], y)
    wsb = mb.mamba_scan_workspace_size(dims)
    ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device=dev) if wsb else None

    def run(i):
        g = sets[i % nsets]
        mb.scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"], True,
                    y=y, last_state=last, stream=stream, workspace=ws)

    ms, clk = time_launches(torch, stream, run, steps, 3, local)
    ms = max_over_ranks(ms, world, dev)
    nb = scan_bytes(w.batch, w.dim, w.dstate, w.seqlen, es, 4)
    gbs = nb / (ms * 1e-3) / 1e9
    rc, pl = mb.mamba_scan_choose_plan(dims)
    plan = [pl.lanes_per_channel, pl.chunks_per_lane, pl.poly8, pl.engine] if rc == mb.MS_OK else None
    out = {"workload": w.name, "ms": ms, "bytes": nb, "value": gbs, "unit": "GB/s",
           "gct_per_s": w.channel_tokens / (ms * 1e-3) / 1e9, "frac": gbs / peak,
           "frac_of_nominal": gbs / NOMINAL_HBM_GBS, "traffic": recorded_traffic(traffic_key),
           "plan": plan, "split_workspace_bytes": wsb,
           "l2": f"{nsets} rotating input sets of {nb / 1e6:.0f} MB (> 126 MB L2)",
           "timing": f"mean of {steps} per-launch event pairs", "clocks": clk}
    del sets, y, last, ws
    torch.cuda.empty_cache()
    return out


# ----------------------------------------------------------- CPU baseline ----

def oracle_sample_time(inp, n_batch_rows, nthreads):
    """Run the fp64 oracle (as it stands) on the first n_batch_rows batch rows
    of the workload; returns (channel_tokens, seconds)."""
    import oracle

    def f64(t):
        return t.to("cpu").to(__import__("torch").float64).numpy()

    sl = slice(0, n_batch_rows)
    args = (f64(inp["u"][sl]), f64(inp["delta"][sl]), f64(inp["A"]), f64(inp["B"][sl]),
            f64(inp["C"][sl]), f64(inp["D"]), f64(inp["z"][sl]), f64(inp["delta_bias"]))
    lib = oracle.load_oracle()
    t = time.perf_counter()
    oracle.scan(*args, softplus_flag=True, lib=lib, nthreads=nthreads)
    dt = time.perf_counter() - t
    b, d, L = inp["u"][sl].shape
    return b * d * L, dt


def cpu_threads():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


# ------------------------------------------------------------------- main ----

def run_reference(args, w, world, rank):
    """The oracle on the host cores, each step a bounded sample (one batch
    row) of the same workload."""
    if rank != 0:
        return 0
    import torch
    from selective_state_space_40_b200 import synthetic as syn
    torch.set_num_threads(max(1, cpu_threads()))
    inp = syn.scan_inputs(w)
    es = 2 if w.in_dtype == torch.bfloat16 else 4
    threads = cpu_threads()
    rows = 1
    for _ in range(args.warmup):
        oracle_sample_time(inp, rows, threads)
    total_ct, total_s = 0, 0.0
    for _ in range(args.steps):
        ct, s = oracle_sample_time(inp, rows, threads)
        total_ct += ct
        total_s += s
    ct_s = total_ct / total_s
    bytes_per_ct = scan_bytes(w.batch, w.dim, w.dstate, w.seqlen, es, 4) / w.channel_tokens
    gbs = ct_s * bytes_per_ct / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s",
        "gct_per_s": ct_s / 1e9, "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total_s / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "dim": w.dim, "dstate": w.dstate,
                   "seqlen": w.seqlen, "in_dtype": "bf16", "out_dtype": "f64",
                   "sample": f"{rows} of {w.batch} batch rows per step"},
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": f"{rows} of {w.batch} batch rows ({rows * w.dim * w.seqlen} channel-tokens) per step"},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world, rank, local = dist_env()
    from selective_state_space_40_b200 import synthetic as syn
    w = syn.M130

    if args.impl == "reference":
        return run_reference(args, w, world, rank)

    import torch
    from selective_state_space_40_b200 import binding as mb
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist(world, "nccl")
    if mb.mamba_device_check() != mb.MS_OK:
        raise SystemExit("libmambascan: " + mb.mamba_status_string(mb.mamba_device_check()))

    es = 2 if w.in_dtype == torch.bfloat16 else 4
    host = syn.scan_inputs(w)
    NSETS = 3
    sets = [{k: v.to(dev) for k, v in host.items()} for _ in range(NSETS)]
    y = torch.empty(w.batch, w.dim, w.seqlen, dtype=torch.float32, device=dev)
    y_alt = torch.empty_like(y)
    last = torch.empty(w.batch, w.dim, w.dstate, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(i):
        g = sets[i % NSETS]
        mb.scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"], g["delta_bias"],
                    True, y=y if i & 1 == 0 else y_alt, last_state=last, stream=stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()

    # ---- timed region: K steps, per-launch events on the launching stream
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local, period=0.001) as clk:
        t0.record(stream)
        for i in range(args.steps):
            ev[i][0].record(stream)
            step(i)
            ev[i][1].record(stream)
        t1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    elapsed_ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
    kernel_ms = statistics.fmean(a.elapsed_time(b) for a, b in ev)
    kernel_ms = max_over_ranks(kernel_ms, world, dev)

    nbytes = scan_bytes(w.batch, w.dim, w.dstate, w.seqlen, es, 4)
    ct = w.channel_tokens
    value = world * nbytes * args.steps / (elapsed_ms * 1e-3) / 1e9
    gct = world * ct * args.steps / (elapsed_ms * 1e-3) / 1e9
    peak, peak_kind = measured_peaks()
    achieved = nbytes / (kernel_ms * 1e-3) / 1e9
    traffic = recorded_traffic("scan_fwd_130m")
    main_dims = mb.scan_dims_for(sets[0]["u"], sets[0]["delta"], sets[0]["B"], sets[0]["C"], sets[0]["z"], y)
    prc, mpl = mb.mamba_scan_choose_plan(main_dims)
    main_kernel = ("scan_fwd_tmem_kernel" if prc == mb.MS_OK and mpl.engine == mb.MS_ENGINE_TMEM
                   else "scan_fwd_kernel")

    # ---- end to end through the public API with host buffers: every step
    # copies its inputs from pinned host memory, scans, and copies y and
    # last_state back. Steps are pipelined over three streams (host->device,
    # compute, device->host) with two device buffer sets, so step i's upload,
    # step i-1's scan and step i-2's download overlap (the two copy directions
    # are independent links).
    pinned = {k: v.pin_memory() for k, v in host.items()}
    y_host = [torch.empty(y.shape, dtype=y.dtype, pin_memory=True) for _ in range(2)]
    last_host = [torch.empty(last.shape, dtype=last.dtype, pin_memory=True) for _ in range(2)]
    ys = [y, torch.empty_like(y)]
    lasts = [last, torch.empty_like(last)]
    h2d = sum(v.numel() * v.element_size() for v in pinned.values())
    d2h = y_host[0].numel() * 4 + last_host[0].numel() * 4
    # at least 12 pipelined steps (about 40 ms), so the first upload and the last
    # download weigh little against the steady state
    e2e_steps = max(12, min(40, args.steps // 10))
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()  # noqa: E731
    in_done, comp_done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]

    def e2e_run(n):
        for i in range(n):
            k = i & 1
            d_in = sets[k]  # two of the device sets serve as the e2e buffers
            if i >= 2:
                s_in.wait_event(comp_done[k])       # the scan of step i-2 has read these inputs
            with torch.cuda.stream(s_in):
                for name, v in pinned.items():
                    d_in[name].copy_(v, non_blocking=True)
            in_done[k].record(s_in)
            stream.wait_event(in_done[k])
            if i >= 2:
                stream.wait_event(out_done[k])      # step i-2's outputs have left the device
            mb.scan_fwd(d_in["u"], d_in["delta"], d_in["A"], d_in["B"], d_in["C"], d_in["D"], d_in["z"],
                        d_in["delta_bias"], True, y=ys[k], last_state=lasts[k], stream=stream)
            comp_done[k].record(stream)
            s_out.wait_event(comp_done[k])
            with torch.cuda.stream(s_out):
                y_host[k].copy_(ys[k], non_blocking=True)
                last_host[k].copy_(lasts[k], non_blocking=True)
            out_done[k].record(s_out)

    e2e_run(2)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    e2e_run(e2e_steps)
    e1.record(s_out)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    e2e_gbs = world * nbytes * e2e_steps / (e2e_ms * 1e-3) / 1e9

    # ---- decode step (selective state update) at b256 d5120 N16: back-to-back
    # steps over three rotating state buffers (3 x 84 MB > 126 MB L2), the
    # steady state of generation where each layer's state is cold when its
    # next token comes.
    dw = syn.DECODE
    dp = {k: v.to(dev) for k, v in syn.decode_params(dw).items()}
    ds = {k: v.to(dev) for k, v in syn.decode_step_inputs(dw, 0).items()}
    states = [dp["state0"].clone() for _ in range(3)]
    yd = torch.empty(dw.batch, dw.dim, dtype=torch.float32, device=dev)

    def dec(i):
        mb.state_update(states[i % 3], ds["x"], ds["delta"], dp["A"], ds["B"], ds["C"], dp["D"], ds["z"],
                        dp["delta_bias"], True, y=yd, stream=stream)

    for i in range(6):
        dec(i)
    dec_steps = 60
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    d0.record(stream)
    for i in range(dec_steps):
        dec(i)
    d1.record(stream)
    torch.cuda.synchronize()
    dec_ms = max_over_ranks(d0.elapsed_time(d1) / dec_steps, world, dev)
    dbytes = decode_bytes(dw.batch, dw.dim, dw.dstate, 2, 4)
    dec_gbs = dbytes / (dec_ms * 1e-3) / 1e9
    del states

    # ---- the other forward workloads: the 2.8B-class layer (two rotating
    # 842 MB input sets) and the long-context fp32 layer (4.3 GB per launch,
    # sequence split in segments; one input set is far above L2)
    del sets[2:]
    fwd_2p8b = forward_leg(torch, mb, syn, syn.M2P8, stream, dev, local, world, peak, 30, 2, "scan_fwd_2p8b")
    fwd_long = forward_leg(torch, mb, syn, syn.LONG, stream, dev, local, world, peak, 8, 1, "scan_fwd_long")

    # ---- scan with the causal conv front-end (width 4) on the same layer: u is
    # formed from the conv input x in the load stage, so the bytes are the
    # scan's plus the filter.
    cp = {k: v.to(dev) for k, v in syn.conv_params(w, 4).items()}
    conv_steps = 40

    def conv_step(i):
        g = sets[i & 1]
        mb.conv_scan_fwd(g["u"], cp["conv_w"], g["delta"], g["A"], g["B"], g["C"], g["D"], g["z"],
                         g["delta_bias"], True, conv_b=cp["conv_b"], y=y, last_state=last, stream=stream)

    for i in range(4):
        conv_step(i)
    cev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(conv_steps)]
    torch.cuda.synchronize()
    for i in range(conv_steps):
        cev[i][0].record(stream)
        conv_step(i)
        cev[i][1].record(stream)
    torch.cuda.synchronize()
    conv_ms = max_over_ranks(statistics.fmean(a.elapsed_time(b) for a, b in cev), world, dev)
    conv_bytes = nbytes + w.dim * 5 * 4
    conv_gbs = conv_bytes / (conv_ms * 1e-3) / 1e9

    # ---- training step of the scan on the same layer: forward with saved
    # states, then the backward from them (dout N(0,1) fp32)
    gdo = torch.Generator().manual_seed(77)
    dout = torch.randn(w.batch, w.dim, w.seqlen, generator=gdo).to(dev)
    g0 = sets[0]
    bwd_steps = 10
    # the pairs are queued back to back and synchronized once, so the host's
    # call of the next pair overlaps the device's work and no event window
    # holds an idle device waiting for a launch
    pairs = []
    torch.cuda.synchronize()
    for i in range(2 + bwd_steps):
        f0, f1, b1 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        f0.record(stream)
        _, _, ck = mb.scan_fwd_train(g0["u"], g0["delta"], g0["A"], g0["B"], g0["C"], g0["D"], g0["z"],
                                     g0["delta_bias"], True, stream=stream)
        f1.record(stream)
        mb.scan_bwd(g0["u"], g0["delta"], g0["A"], g0["B"], g0["C"], g0["D"], g0["z"], g0["delta_bias"], True,
                    dout, ckpt=ck, stream=stream)
        b1.record(stream)
        if i >= 2:
            pairs.append((f0, f1, b1))
    torch.cuda.synchronize()
    fwd_train_ms = max_over_ranks(statistics.fmean(f0.elapsed_time(f1) for f0, f1, _ in pairs), world, dev)
    bwd_ms = max_over_ranks(statistics.fmean(f1.elapsed_time(b1) for _, f1, b1 in pairs), world, dev)
    bbytes = bwd_bytes(w.batch, w.dim, w.dstate, w.seqlen, es, 4)
    del dout

    # ---- Mamba-2 SSD layer (2.7B-class): chunked matrix view on the tensor cores
    sw = syn.SSD_2P7B
    ssd_in = [{k: v.to(dev) for k, v in syn.ssd_inputs(sw).items()} for _ in range(2)]
    ssd_y = torch.empty(sw.batch, sw.seqlen, sw.nheads, sw.headdim, dtype=torch.float32, device=dev)
    ssd_steps = 20
    sdims = mb.SsdDims(sw.batch, sw.seqlen, sw.nheads, sw.headdim, sw.dstate, sw.ngroups, *ssd_in[0]["x"].stride()[:3],
                       *ssd_in[0]["dt"].stride()[:2], *ssd_in[0]["B"].stride()[:3], *ssd_in[0]["C"].stride()[:3],
                       *ssd_y.stride()[:3], mb.MS_BF16, mb.MS_F32)
    ssd_ws = torch.empty(mb.mamba2_ssd_workspace_size(sdims), dtype=torch.uint8, device=dev)

    def ssd_step(i):
        g = ssd_in[i & 1]
        mb.ssd_fwd(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], g["dt_bias"], True, y=ssd_y,
                   return_final_state=False, stream=stream, workspace=ssd_ws)

    for i in range(3):
        ssd_step(i)
    sev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(ssd_steps)]
    torch.cuda.synchronize()
    for i in range(ssd_steps):
        sev[i][0].record(stream)
        ssd_step(i)
        sev[i][1].record(stream)
    torch.cuda.synchronize()
    ssd_ms = max_over_ranks(statistics.fmean(a.elapsed_time(b) for a, b in sev), world, dev)
    sbytes = ssd_bytes(sw.batch, sw.seqlen, sw.nheads, sw.headdim, sw.dstate, sw.ngroups, 2, 4) \
        - sw.batch * sw.nheads * sw.headdim * sw.dstate * 4  # no final state requested
    sflops = ssd_flops(sw.batch, sw.seqlen, sw.nheads, sw.headdim, sw.dstate, chunk=128)
    del ssd_in, ssd_ws

    # ---- Mamba-2 SSD decode step (2.7B-class layer, 64 sequences): the fp32
    # state [64, 80, 64, 128] (168 MB) read and written once per step; two
    # states rotate (336 MB > L2)
    ub, uH, uP, uN = 64, sw.nheads, sw.headdim, sw.dstate
    gsd = torch.Generator().manual_seed(11)
    ust = [(0.1 * torch.randn(ub, uH, uP, uN, generator=gsd)).to(dev) for _ in range(2)]
    ux = torch.randn(ub, uH, uP, generator=gsd).to(torch.bfloat16).to(dev)
    udt = torch.randn(ub, uH, generator=gsd).to(torch.bfloat16).to(dev)
    uB = torch.randn(ub, 1, uN, generator=gsd).to(torch.bfloat16).to(dev)
    uC = torch.randn(ub, 1, uN, generator=gsd).to(torch.bfloat16).to(dev)
    upar = {k: v.to(dev) for k, v in syn.ssd_inputs(syn.SsdWorkload("p", 1, 1, uH, uP, uN, 1)).items()}
    uy = torch.empty(ub, uH, uP, dtype=torch.float32, device=dev)

    def ssd_dec(i):
        mb.ssd_state_update(ust[i & 1], ux, udt, upar["A"], uB, uC, upar["D"], upar["dt_bias"], True, y=uy,
                            stream=stream)

    for i in range(4):
        ssd_dec(i)
    u0, u1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    u0.record(stream)
    for i in range(40):
        ssd_dec(i)
    u1.record(stream)
    torch.cuda.synchronize()
    ssd_dec_ms = max_over_ranks(u0.elapsed_time(u1) / 40, world, dev)
    udbytes = ub * uH * uP * uN * 8 + ub * uH * uP * (2 + 4) + ub * uH * 2 + ub * 2 * uN * 2 + 3 * uH * 4
    del ust

    # ---- CPU baseline: the oracle on this host's cores, whole passes over the
    # workload repeated until about ten seconds of wall time have gone by
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        threads = cpu_threads()
        cts, secs, passes = 0, 0.0, 0
        while secs < 10.0 and passes < 50:
            c, s_ = oracle_sample_time(host, w.batch, threads)
            cts, secs, passes = cts + c, secs + s_, passes + 1
        ct_s = cts / secs
        cpu = {"value": ct_s * nbytes / ct / 1e9, "unit": "GB/s", "gct_per_s": ct_s / 1e9,
               "cores": threads, "kind": "oracle",
               "sample": f"{passes} full passes over the workload ({cts} channel-tokens), "
                         f"{secs:.1f} s wall on {threads} threads"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "gct_per_s": gct,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": w.name, "batch": w.batch, "dim": w.dim, "dstate": w.dstate,
                       "seqlen": w.seqlen, "in_dtype": "bf16", "out_dtype": "f32",
                       "parallelism": f"dp{world}" if world > 1 else "single",
                       "l2": "three rotating input sets of 254 MB each and two y buffers (> 126 MB L2), no flush"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "peak_source": f"{peak_kind} hbm_gbs (copy, burst)",
                         "kernel": main_kernel, "bytes_per_launch": nbytes,
                         "kernel_ms": kernel_ms, "nominal_peak": NOMINAL_HBM_GBS,
                         "frac_of_nominal": achieved / NOMINAL_HBM_GBS,
                         "traffic_over_bytes": None if traffic is None else traffic / nbytes},
            "e2e": {"value": e2e_gbs, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                    "pipelining": "upload, scan and download of consecutive steps overlap on three streams"},
            "scan_2p8b": fwd_2p8b,
            "scan_long": fwd_long,
            "decode_step": {"workload": dw.name, "value": dec_gbs, "unit": "GB/s",
                            "ms": dec_ms, "bytes": dbytes, "frac": dec_gbs / peak,
                            "frac_of_nominal": dec_gbs / NOMINAL_HBM_GBS,
                            "l2": "back-to-back steps over 3 rotating 84 MB states (> 126 MB L2)",
                            "timing": f"one event pair around {dec_steps} back-to-back launches",
                            "traffic": recorded_traffic("decode_step")},
            "conv_scan": {"workload": w.name + " + causal conv width 4", "value": conv_gbs, "unit": "GB/s",
                          "ms": conv_ms, "bytes": conv_bytes, "frac": conv_gbs / peak,
                          "l2": "two rotating input sets", "timing": "mean of per-launch event pairs",
                          "traffic": recorded_traffic("conv_scan_130m")},
            "backward": {"workload": w.name + ", dout N(0,1) fp32", "fwd_train_ms": fwd_train_ms,
                         "bwd_ms": bwd_ms, "bwd_bytes": bbytes, "value": bbytes / (bwd_ms * 1e-3) / 1e9,
                         "unit": "GB/s", "frac": bbytes / (bwd_ms * 1e-3) / 1e9 / peak,
                         "timing": f"mean of {bwd_steps} event-timed (forward with saved states, backward) pairs, queued back to back",
                         "traffic": recorded_traffic("scan_bwd_130m")},
            "ssd": {"workload": sw.name, "ms": ssd_ms, "bytes": sbytes,
                    "value": sbytes / (ssd_ms * 1e-3) / 1e9, "unit": "GB/s",
                    "frac_hbm": sbytes / (ssd_ms * 1e-3) / 1e9 / peak,
                    "tflops": sflops / (ssd_ms * 1e-3) / 1e12, "algorithmic_flops": sflops,
                    "frac_tensor": sflops / (ssd_ms * 1e-3) / 1e12 / measured_bf16_tflops(),
                    "bound": ssd_bound(sbytes, sflops, peak, measured_bf16_tflops()),
                    "timing": "mean of per-launch event pairs, two rotating input sets",
                    "traffic": recorded_traffic("ssd_2p7b")},
            "ssd_decode": {"workload": "mamba2-2.7b-class decode b64 H80 P64 N128 bf16, fp32 state",
                           "ms": ssd_dec_ms, "bytes": udbytes, "value": udbytes / (ssd_dec_ms * 1e-3) / 1e9,
                           "unit": "GB/s", "frac": udbytes / (ssd_dec_ms * 1e-3) / 1e9 / peak,
                           "timing": "one event pair around 40 back-to-back steps over two rotating states",
                           "traffic": recorded_traffic("ssd_decode")},
            "gpu_launches": args.steps,
            "clocks": clk.summary(),
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
