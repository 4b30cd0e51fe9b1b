#!/usr/bin/env python
"""Benchmark: FourTune W4A4G4 triple-branch linear, forward + backward, on B200.

One step = fourtune_linear_fwd + fourtune_linear_bwd (every kernel of the hot
path: fused X pass, FP4 GEMM + up-projection, fused G pass, FP4 dX GEMM, dA and
dB) on the FLUX-width layer: M = 4608 tokens, K = N = 3072, stabilizer
rank 32, LoRA rank 32, seeded synthetic bf16 data (synth.py).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  `value` is device time from CUDA events summed
over exactly K steps (L2 flushed before each step, outside the events, by a
256 MB write followed by a 256 MB read of another buffer), max over ranks, with
no event between the kernels of a step; that block of K steps is repeated back
to back for ~0.4 s (the clock sampler's window) and the median block counts; K further steps with an event pair
around every kernel give the per-kernel times (`kernels`, `roofline`);
`e2e` runs K steps through the same C ABI with
inputs in pinned host memory: every step copies its X and dY host -> device and
its dA and dB device -> host inside one timed region, the way a training loop
feeds the layer -- the next step's inputs are copied on a second stream into a
second device buffer while the current step computes, the forward starts when
its X has landed and the backward when its dY has.  `--impl reference` times the CPU oracle on a bounded sample of
the same workload.  With N > 1 (torchrun) every rank runs an independent
replica: the layer has no data-path exchange.
"""
import argparse
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

WORKLOAD = "flux-linear-3072"
METRIC = "W4A4G4 linear fwd+bwd TFLOPS & tokens/s on 1 B200; % of dense FP4 peak"
FALLBACK = dict(hbm_gbs=6650.0, bf16_tflops=1590.0)
FP4_PER_BF16 = 4.0          # nominal dense ratio 9 PF / 2.25 PF
ORACLE_ROWS = 256           # rows of the workload per CPU-oracle sample
CLOCK_WINDOW_S = 0.4        # repeats of the timed block fill about this long (clock record)


def layer_work(M, K, N, r_s, r):
    """FP4 GEMM FLOPs (forward + dX; no weight gradient) and bf16 low-rank FLOPs per step."""
    R = r_s + r
    fp4 = 4 * M * N * K
    lowrank = 4 * M * R * (K + N) + 2 * M * r * (K + N)
    return fp4, lowrank


def kernel_work(M, K, N, r_s, r):
    """Algorithmic work per launch of each kernel: ('tensor', FLOPs) or ('hbm', bytes)."""
    R = r_s + r
    return {
        "fwd.xpass_quant_down": ("hbm", 2 * M * K + M * K // 2 + M * K // 256 + 2 * M * R),
        "fwd.gemm_fp4_fwd": ("tensor", 2 * M * N * K),
        "bwd.gpass_quant_down": ("hbm", 2 * M * N + M * N // 2 + M * N // 256 + 2 * M * R),
        "bwd.gemm_fp4_dx": ("tensor", 2 * M * N * K),
        "bwd.tgrad_dA_dB": ("hbm", 2 * M * K + 2 * M * N + 4 * M * R + 4 * (K + N) * r),
    }


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    bf16_tflops_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    except Exception:
        return dict(hbm_gbs=FALLBACK["hbm_gbs"], bf16_tflops=FALLBACK["bf16_tflops"],
                    bf16_tflops_sustained=FALLBACK["bf16_tflops"], source="fallback")


# ------------------------------------------------------------------ clocks
_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
            0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
            0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}


class ClockSampler:
    """Reads SM clock and clock-event reasons through NVML every ~2 ms (read-only)."""

    def __init__(self, index, period=0.002):
        self.period = period
        self.samples, self.reasons, self.max_mhz = [], 0, None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self._nv:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        if self._thread:
            self._stop.set()
            self._thread.join()
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "samples": len(self.samples),
                "reasons": [n for b, n in _REASONS.items() if self.reasons & b]}


# ------------------------------------------------------------------ oracle (CPU)
def oracle_step(p, Rc, Rs, X, dY):
    from oracle import layer as olayer
    f = olayer.linear_fwd(X, Rc, Rs, p["S_dn"], p["S_up"], p["A"], p["B"], p.get("bias"))
    b = olayer.linear_bwd(dY, X, f["L"], Rc, Rs, p["S_dn"], p["S_up"], p["A"], p["B"])
    return f, b


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count()


def oracle_inputs(rows):
    from bit_lora_fine_b200 import synth
    from oracle import block16
    wl = synth.WORKLOADS[WORKLOAD]
    spec = wl.layers[0]
    p = synth.layer_params(spec)
    Rc, Rs = block16.quantize(p["R"])                    # frozen weight: quantized once, outside timing
    X = synth.layer_input(wl)[:rows]
    dY = synth.upstream_grad(wl)[:rows]
    return wl, spec, p, Rc, Rs, X, dY


def time_oracle(rows, repeats=1):
    """Times the CPU oracle on the first `rows` tokens; returns (times, FLOPs, outputs)."""
    wl, spec, p, Rc, Rs, X, dY = oracle_inputs(rows)
    times = []
    out = None
    for _ in range(repeats):
        t0 = time.perf_counter()
        out = oracle_step(p, Rc, Rs, X, dY)
        times.append(time.perf_counter() - t0)
    fp4, lr = layer_work(rows, spec.K, spec.N, spec.r_s, spec.r)
    return times, (fp4 + lr), out


def parity_record(ref, ft, lay, X, dY, ws_f, ws_b, Y, dX):
    """The timed configuration's parity against the oracle on the whole workload:
    one more fwd+bwd with fp32 outputs (outside any timing) gives the max-normwise
    error max|g - r| / max|r| of y, dX, dA, dB (the tolerance's definition), and the
    timed step's bf16 y and dX must equal the nearest-even rounding of those fp32
    outputs bit for bit."""
    import torch
    f, b = ref
    Y32, L32, _ = ft.linear_fwd(lay, X, torch.float32, ws=ws_f)
    dX32, dA32, dB32, _ = ft.linear_bwd(lay, dY, X, L32, torch.float32, ws=ws_b)
    torch.cuda.synchronize()
    host = lambda t: t.float().cpu().numpy().astype(np.float64)
    nw = lambda g, r: float(np.abs(g - r).max() / np.abs(r).max())
    return {"y": nw(host(Y32), f["y"]), "dX": nw(host(dX32), b["dX"]), "dA": nw(host(dA32), b["dA"]),
            "dB": nw(host(dB32), b["dB"]),
            "bf16_outputs_are_rne_of_fp32": bool(torch.equal(Y, Y32.to(torch.bfloat16)) and
                                                 torch.equal(dX, dX32.to(torch.bfloat16))),
            "note": "max-normwise error of fp32 outputs vs the CPU oracle on the whole workload; "
                    "the timed step's bf16 outputs checked as their nearest-even rounding"}


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    from bit_lora_fine_b200 import synth
    spec = synth.WORKLOADS[WORKLOAD].layers[0]
    wl, spec, p, Rc, Rs, X, dY = oracle_inputs(ORACLE_ROWS)
    for _ in range(args.warmup):
        oracle_step(p, Rc, Rs, X, dY)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(p, Rc, Rs, X, dY)
    dt = time.perf_counter() - t0
    fp4, lr = layer_work(ORACLE_ROWS, spec.K, spec.N, spec.r_s, spec.r)
    value = (fp4 + lr) * args.steps / dt / 1e12
    sample = f"{ORACLE_ROWS} of {wl.M} tokens per step, full K=N={spec.K}, ranks {spec.r_s}/{spec.r}"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "tokens_per_s": ORACLE_ROWS * args.steps / dt,
        "config": {"workload": WORKLOAD, "M": wl.M, "K": spec.K, "N": spec.N, "r_s": spec.r_s, "r": spec.r},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ replicas
def max_over_ranks(values, device):
    """Element-wise maximum of a list of floats over all ranks (every rank
    gets it); identity on one process.  Timing is the slowest replica's."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_throughput(work_per_step, steps, world, ms):
    """Whole-job throughput (work units per second) of `world` replicas that
    each ran `steps` steps of `work_per_step` in `ms` milliseconds (the
    maximum over ranks): per-GPU work is fixed, so this is weak scaling."""
    return work_per_step * steps * world / (ms / 1e3)


# ------------------------------------------------------------------ ours (GPU)
def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from bit_lora_fine_b200 import fourtune as ft
    from bit_lora_fine_b200 import synth

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = synth.WORKLOADS[WORKLOAD]
    spec = wl.layers[0]
    M, K, N, r_s, r = wl.M, spec.K, spec.N, spec.r_s, spec.r
    p = synth.layer_params(spec)
    X_h = synth.layer_input(wl)
    dY_h = synth.upstream_grad(wl)
    up = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev).to(torch.bfloat16)
    lay = ft.Linear.from_weights(up(p["R"]), up(p["S_dn"]), up(p["S_up"]), up(p["A"]), up(p["B"]))
    X, dY = up(X_h), up(dY_h)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    L = torch.empty((M, r_s + r), dtype=torch.bfloat16, device=dev)
    dX = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    dA = torch.zeros((K, r), dtype=torch.float32, device=dev)
    dB = torch.zeros((r, N), dtype=torch.float32, device=dev)
    ws_f, ws_b = lay.fwd_workspace(M), lay.bwd_workspace(M)
    # L2 flush before every step: write 256 MB (> 126 MB L2), then read another
    # 256 MB so that no input of the step is cached and no dirty line is left
    # for the step's reads to write back
    flush_w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(64 << 20, dtype=torch.float32, device=dev)

    class _Flush:
        def zero_(self):
            flush_w.zero_()
            flush_r.sum()
    flush = _Flush()

    nf, nb = len(ft.FWD_KERNELS), len(ft.BWD_KERNELS)
    names = [f"fwd.{k}" for k in ft.FWD_KERNELS] + [f"bwd.{k}" for k in ft.BWD_KERNELS]

    def mk_events(n):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        for e in evs:
            e.record()                     # materialize the CUDA event
        return evs

    def step(evf=None, evb=None):
        ft.linear_fwd(lay, X, ws=ws_f, Y=Y, L=L, events=evf)
        ft.linear_bwd(lay, dY, X, L, ws=ws_b, dX=dX, dA=dA, dB=dB, events=evb)

    for _ in range(max(args.warmup, 1)):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    t_w = time.perf_counter()                      # wall time of a warm step (flush included)
    for _ in range(5):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    wall_per_step = (time.perf_counter() - t_w) / 5
    ft.device_status(ws_f)
    ft.device_status(ws_b)

    # timed region: K steps with no event between the kernels of a step (the
    # kernels chain through programmatic dependent launch), timed as one block
    # between a barrier and a synchronize on both sides.  The block is repeated
    # back to back (the same K steps each time) for ~0.4 s so that the clock
    # sampler sees the GPU under load; the value is the median block.  Then K
    # more steps with an event pair around every kernel, for the breakdown.
    reps = int(min(200, max(3, np.ceil(CLOCK_WINDOW_S / max(args.steps * wall_per_step, 1e-6)))))
    blocks = [[mk_events(2) for _ in range(args.steps)] for _ in range(reps)]
    ksteps = [(mk_events(2 * nf), mk_events(2 * nb)) for _ in range(args.steps)]
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank)
    clocks.start()
    for steps in blocks:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        for se in steps:
            flush.zero_()
            se[0].record()
            step()
            se[1].record()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
    torch.cuda.synchronize()
    clk = clocks.stop()
    block_ms = [sum(se[0].elapsed_time(se[1]) for se in steps) for steps in blocks]
    for evf, evb in ksteps:
        flush.zero_()
        step(evf, evb)
    torch.cuda.synchronize()
    ft.device_status(ws_f)
    ft.device_status(ws_b)

    total_ms = float(statistics.median(block_ms))
    per_kernel = {n: 0.0 for n in names}
    for evf, evb in ksteps:
        for i in range(nf):
            per_kernel[names[i]] += evf[2 * i].elapsed_time(evf[2 * i + 1])
        for i in range(nb):
            per_kernel[names[nf + i]] += evb[2 * i].elapsed_time(evb[2 * i + 1])

    # ---- end to end through the C ABI with host-resident inputs and outputs:
    # double-buffered device inputs, H2D copies on their own stream one step
    # ahead, D2H of the gradients on the compute stream
    X_pin = torch.from_numpy(synth.bf16_bits(X_h).view(np.int16)).pin_memory()
    dY_pin = torch.from_numpy(synth.bf16_bits(dY_h).view(np.int16)).pin_memory()
    dA_pin = torch.empty((K, r), dtype=torch.float32).pin_memory()
    dB_pin = torch.empty((r, N), dtype=torch.float32).pin_memory()
    Xb = [X, torch.empty_like(X)]
    dYb = [dY, torch.empty_like(dY)]
    main_s = torch.cuda.current_stream()
    copy_s = torch.cuda.Stream()

    def e2e_run(nsteps):
        evx = [torch.cuda.Event() for _ in range(nsteps)]
        evy = [torch.cuda.Event() for _ in range(nsteps)]
        done = [torch.cuda.Event() for _ in range(nsteps)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(main_s)
        copy_s.wait_stream(main_s)

        def h2d(k):
            b = k % 2
            with torch.cuda.stream(copy_s):
                if k >= 2:
                    copy_s.wait_event(done[k - 2])          # step k-2 has finished with this buffer
                Xb[b].view(torch.int16).copy_(X_pin, non_blocking=True)
                evx[k].record(copy_s)
                dYb[b].view(torch.int16).copy_(dY_pin, non_blocking=True)
                evy[k].record(copy_s)

        h2d(0)
        for k in range(nsteps):
            if k + 1 < nsteps:
                h2d(k + 1)
            b = k % 2
            main_s.wait_event(evx[k])
            ft.linear_fwd(lay, Xb[b], ws=ws_f, Y=Y, L=L)
            main_s.wait_event(evy[k])
            ft.linear_bwd(lay, dYb[b], Xb[b], L, ws=ws_b, dX=dX, dA=dA, dB=dB)
            dA_pin.copy_(dA, non_blocking=True)
            dB_pin.copy_(dB, non_blocking=True)
            done[k].record(main_s)
        main_s.wait_stream(copy_s)
        t1.record(main_s)
        return t0, t1

    e2e_run(max(args.warmup, 1))
    torch.cuda.synchronize()
    t0, t1 = e2e_run(args.steps)
    torch.cuda.synchronize()
    e2e_ms = t0.elapsed_time(t1)

    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], dev)

    fp4, lr = layer_work(M, K, N, r_s, r)
    sec = total_ms / 1e3
    value = job_throughput(fp4 + lr, args.steps, world, total_ms) / 1e12
    peaks = load_peaks()
    fp4_peak = peaks["bf16_tflops"] * FP4_PER_BF16
    work = kernel_work(M, K, N, r_s, r)
    kern = {}
    for n in names:
        avg_ms = per_kernel[n] / args.steps
        kind, amount = work[n]
        if kind == "tensor":
            ach = amount / (avg_ms / 1e3) / 1e12
            kern[n] = {"us": avg_ms * 1e3, "achieved": ach, "unit": "TFLOP/s", "frac": ach / fp4_peak}
        else:
            ach = amount / (avg_ms / 1e3) / 1e9
            kern[n] = {"us": avg_ms * 1e3, "achieved": ach, "unit": "GB/s", "frac": ach / peaks["hbm_gbs"]}
    dom = max(names, key=lambda n: per_kernel[n])
    kind, amount = work[dom]
    dk = kern[dom]
    traffic = load_traffic(dom)
    roofline = {"kernel": dom, "bound": kind, "achieved": dk["achieved"],
                "peak": fp4_peak if kind == "tensor" else peaks["hbm_gbs"], "unit": dk["unit"],
                "frac": dk["frac"], "traffic": traffic,
                "peak_source": ("FP4 = measured bf16 burst x 4 (nominal dense ratio)" if kind == "tensor"
                                else "measured HBM copy") + f" ({peaks['source']})",
                "algorithmic_per_launch": amount}

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4(e2m1 x e2m1, e4m3 16x16 scales)->f32; bf16 low-rank",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "M": M, "K": K, "N": N, "r_s": r_s, "r": r, "global_batch_tokens": M * world,
                   "l2": "flushed before each step outside the timed events: 256 MB write, then 256 MB read of "
                         "another buffer (no input cached, no dirty lines)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single"},
        "tokens_per_s": M * args.steps * world / sec,
        "fp4_tflops": fp4 * args.steps * world / sec / 1e12,
        "fp4_peak_frac": fp4 * args.steps * world / sec / 1e12 / fp4_peak,
        "fp4_peak_tflops": fp4_peak,
        "e2e": {"value": job_throughput(fp4 + lr, args.steps, world, e2e_ms) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": 2 * M * K + 2 * M * N, "d2h_bytes_per_step": 4 * K * r + 4 * r * N},
        "gpu_launches": args.steps * (nf + nb + 2),   # + each call's workspace-header clear
        "kernel_breakdown": "per-kernel times from K separate steps with an event pair around every kernel; "
                            "those steps run every kernel on all SMs one after another, the timed steps run "
                            "dA/dB on a second stream beside the dX GEMM",
        "roofline": roofline,
        "kernels": kern,
        "clocks": clk,
        "timed_blocks": {"repeats": reps, "steps_each": args.steps, "median_ms": total_ms,
                         "min_ms": min(block_ms), "max_ms": max(block_ms),
                         "note": "value = the median of back-to-back timed blocks of exactly K steps"},
    }
    if world == 1 and not args.no_extra:
        names = [n for n in args.extra.split(",") if n]
        bad = [n for n in names if n not in EXTRA_WORKLOADS]
        if bad:
            raise SystemExit(f"unknown --extra workload(s) {bad}; choose from {EXTRA_WORKLOADS}")
        line["configs_extra"] = measure_extra(ft, synth, dev, flush, peaks, steps=max(3, min(args.steps, 10)),
                                              warmup=max(1, min(args.warmup, 3)), names=names)
    if world == 1 and not args.no_extra and not args.no_variants:
        v = measure_variants(ft, synth, dev, flush, steps=max(3, min(args.steps, 10)), warmup=max(1, min(args.warmup, 3)))
        ours_ms = total_ms / args.steps
        for rec in v["variants"].values():
            rec["fourtune_speedup"] = rec["ms_per_step"] / ours_ms
        v["note"] = ("fourtune_speedup = variant step time / the fused W4A4G4 step time of this line "
                     "(ms_per_step); the bf16 LoRA layer has no stabilizer (rank-32 adapter only)")
        line["variants"] = v
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        times, flop_s, ref = time_oracle(M, repeats=1)
        t = min(times)
        line["parity"] = parity_record(ref, ft, lay, X, dY, ws_f, ws_b, Y, dX)
        line["cpu_baseline"] = {"value": flop_s / t / 1e12, "unit": "TFLOP/s", "cores": cpu_cores(),
                                "kind": "oracle",
                                "sample": f"one full fwd+bwd of the workload ({M} tokens, K=N={K}), {t:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ other workloads
EXTRA_WORKLOADS = ("flux-mlp-3072", "flux-single-stream", "video-mlp-5120")


def measure_extra(ft, synth, dev, flush, peaks, steps, warmup, names=EXTRA_WORKLOADS):
    """The other workloads (MLP pair, single-stream block linears, video MLP): device
    time of fwd+bwd steps (L2 flushed before each, no events inside), then one step
    with an event pair around every kernel for the breakdown."""
    import torch
    up = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev).to(torch.bfloat16)
    fp4_peak = peaks["bf16_tflops"] * FP4_PER_BF16
    out = {}
    for name in names:
        wl = synth.WORKLOADS[name]
        M = wl.M
        layers = []
        for li, spec in enumerate(wl.layers):
            p = synth.layer_params(spec, li)
            layers.append(ft.Linear.from_weights(up(p["R"]), up(p["S_dn"]), up(p["S_up"]), up(p["A"]), up(p["B"]),
                                                 up(p["bias"]) if p["bias"] is not None else None))
        fp4 = lr = 0
        for spec in wl.layers:
            a, b = layer_work(M, spec.K, spec.N, spec.r_s, spec.r)
            fp4, lr = fp4 + a, lr + b
        if wl.kind == "mlp":
            mlp = ft.MLP(layers[0], layers[1])
            X = up(synth.layer_input(wl))
            dY = up(synth.upstream_grad(wl, layer=1))
            H, N2 = mlp.H, mlp.fc2.N
            fo = (torch.empty((M, N2), dtype=torch.bfloat16, device=dev),
                  torch.empty((M, H), dtype=torch.bfloat16, device=dev),
                  torch.empty((M, mlp.fc1.R_all), dtype=torch.bfloat16, device=dev),
                  torch.empty((M, mlp.fc2.R_all), dtype=torch.bfloat16, device=dev))
            dX = torch.empty((M, mlp.fc1.K), dtype=torch.bfloat16, device=dev)
            grads = (torch.zeros((mlp.fc1.K, mlp.fc1.r), dtype=torch.float32, device=dev),
                     torch.zeros((mlp.fc1.r, mlp.fc1.N), dtype=torch.float32, device=dev),
                     torch.zeros((mlp.fc2.K, mlp.fc2.r), dtype=torch.float32, device=dev),
                     torch.zeros((mlp.fc2.r, mlp.fc2.N), dtype=torch.float32, device=dev))
            wsf, wsb = mlp.fwd_workspace(M), mlp.bwd_workspace(M)
            knames = [f"fwd.{k}" for k in ft.MLP_FWD_KERNELS] + [f"bwd.{k}" for k in ft.MLP_BWD_KERNELS]
            nf = len(ft.MLP_FWD_KERNELS)

            def step(evs=None, mlp=mlp, X=X, dY=dY, fo=fo, dX=dX, grads=grads, wsf=wsf, wsb=wsb, nf=nf):
                ft.mlp_fwd(mlp, X, ws=wsf, out=fo, events=None if evs is None else evs[:2 * nf])
                ft.mlp_bwd(mlp, dY, X, fo[1], fo[2], fo[3], grads=grads, ws=wsb, dX=dX,
                           events=None if evs is None else evs[2 * nf:])
        else:
            specs = wl.layers
            Xs = [up(synth.layer_input(wl, layer=li)) for li in range(len(specs))]
            dYs = [up(synth.upstream_grad(wl, layer=li)) for li in range(len(specs))]
            bufs = []
            for li, lay in enumerate(layers):
                bufs.append(dict(Y=torch.empty((M, lay.N), dtype=torch.bfloat16, device=dev),
                                 L=torch.empty((M, lay.R_all), dtype=torch.bfloat16, device=dev),
                                 dX=torch.empty((M, lay.K), dtype=torch.bfloat16, device=dev),
                                 dA=torch.zeros((lay.K, lay.r), dtype=torch.float32, device=dev),
                                 dB=torch.zeros((lay.r, lay.N), dtype=torch.float32, device=dev),
                                 wsf=lay.fwd_workspace(M), wsb=lay.bwd_workspace(M)))
            per = list(ft.FWD_KERNELS) + list(ft.BWD_KERNELS)
            knames = [f"layer{li}.{k}" for li in range(len(layers)) for k in per]
            nf = len(ft.FWD_KERNELS)

            def step(evs=None, layers=layers, Xs=Xs, dYs=dYs, bufs=bufs, nf=nf, per=per):
                for li, lay in enumerate(layers):
                    b = bufs[li]
                    e = None if evs is None else evs[2 * len(per) * li:2 * len(per) * (li + 1)]
                    ft.linear_fwd(lay, Xs[li], ws=b["wsf"], Y=b["Y"], L=b["L"], events=None if e is None else e[:2 * nf])
                    ft.linear_bwd(lay, dYs[li], Xs[li], b["L"], ws=b["wsb"], dX=b["dX"], dA=b["dA"], dB=b["dB"],
                                  events=None if e is None else e[2 * nf:])
        for _ in range(warmup):
            flush.zero_()
            step()
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for a, b in evs:
            flush.zero_()
            a.record()
            step()
            b.record()
        torch.cuda.synchronize()
        ms = sum(a.elapsed_time(b) for a, b in evs) / steps
        kev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * len(knames))]
        for e in kev:
            e.record()
        flush.zero_()
        step(kev)
        torch.cuda.synchronize()
        kern = {n: round(kev[2 * i].elapsed_time(kev[2 * i + 1]) * 1e3, 1) for i, n in enumerate(knames)}
        out[name] = {
            "M": M, "layers": [[sp.K, sp.N, sp.r_s, sp.r] for sp in wl.layers], "kind": wl.kind, "steps": steps,
            "ms_per_step": ms, "value": (fp4 + lr) / (ms / 1e3) / 1e12, "unit": "TFLOP/s",
            "tokens_per_s": M / (ms / 1e3), "fp4_tflops": fp4 / (ms / 1e3) / 1e12,
            "fp4_peak_frac": fp4 / (ms / 1e3) / 1e12 / fp4_peak, "kernels_us": kern,
        }
        del layers, step
        torch.cuda.empty_cache()
    return out


def measure_variants(ft, synth, dev, flush, steps, warmup):
    """FLUX-width layer (M = 4608, K = N = 3072, ranks 32/32) under the 1x16
    group-wise layout (the granularity ablation), the precision
    variants of the paper's ablation (W4A16G4, W4A4G16, W4A16G16), the standard
    bf16 LoRA layer (bf16 weight, rank-32 adapter, no stabilizer) on this
    library's bf16 tensor-core path and through cuBLAS (torch.matmul), and the
    unfused 4-bit layer (separate quantizer, 4-bit GEMM and cuBLAS low-rank
    products: the form the paper's LoRA fusion replaces).  Device time of fwd+bwd
    steps, L2 flushed before each."""
    import torch
    wl = synth.WORKLOADS[WORKLOAD]
    spec = wl.layers[0]
    M, K, N, r_s, r = wl.M, spec.K, spec.N, spec.r_s, spec.r
    p = synth.layer_params(spec)
    up = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev).to(torch.bfloat16)
    bf = torch.bfloat16
    lay = ft.Linear.from_weights(up(p["R"]), up(p["S_dn"]), up(p["S_up"]), up(p["A"]), up(p["B"]))
    l16 = ft.Linear16.from_linear(lay)
    W, A, B = up(p["R"]), up(p["A"]), up(p["B"])
    lora16 = ft.Linear16.from_bf16_lora(W, A, B)
    X, dY = up(synth.layer_input(wl)), up(synth.upstream_grad(wl))
    R = r_s + r
    Y, L, dX = (torch.empty((M, N), dtype=bf, device=dev), torch.empty((M, R), dtype=bf, device=dev),
                torch.empty((M, K), dtype=bf, device=dev))
    dA, dB = torch.zeros((K, r), device=dev), torch.zeros((r, N), device=dev)
    L0 = torch.empty((M, r), dtype=bf, device=dev)
    wsf, wsb = lay.fwd_workspace(M), lay.bwd_workspace(M)
    wsf16, wsb16 = l16.fwd_workspace(M), l16.bwd_workspace(M)
    wsl_f, wsl_b = lora16.fwd_workspace(M), lora16.bwd_workspace(M)
    D, U = lay.t["D"], lay.t["U"]

    def w4a16g4():
        ft.linear_fwd_a16(l16, X, ws=wsf16, Y=Y, L=L)
        ft.linear_bwd(lay, dY, X, L, ws=wsb, dX=dX, dA=dA, dB=dB)

    def w4a4g16():
        ft.linear_fwd(lay, X, ws=wsf, Y=Y, L=L)
        ft.linear_bwd_g16(l16, dY, X, L, ws=wsb16, dX=dX, dA=dA, dB=dB)

    def w4a16g16():
        ft.linear_fwd_a16(l16, X, ws=wsf16, Y=Y, L=L)
        ft.linear_bwd_g16(l16, dY, X, L, ws=wsb16, dX=dX, dA=dA, dB=dB)

    def lora_bf16_ours():
        ft.linear_fwd_a16(lora16, X, ws=wsl_f, Y=Y, L=L0)
        ft.linear_bwd_g16(lora16, dY, X, L0, ws=wsl_b, dX=dX, dA=dA, dB=dB)

    Wt = W.t()

    def lora_bf16_cublas():
        Lc = X @ A
        Yc = torch.addmm(Lc @ B, X, Wt)
        P = dY @ B.t()
        dXc = torch.addmm(P @ A.t(), dY, W)
        dAc = X.t() @ P
        dBc = Lc.t() @ dY
        return Yc, dXc, dAc, dBc

    R_sf, R_sf_t = lay.t["R_sf"], lay.t["R_sf_t"]
    ws_g = torch.empty(256, dtype=torch.uint8, device=dev)
    r_sl = slice(r_s, R)

    def unfused_w4():
        # forward: quantizer, 4-bit GEMM, then the low-rank branches as separate products
        xc, xs, _ = ft.quantize_block16(X)
        Yu, _ = ft.gemm_block16(xc, ft.mma_scales(xs, M, K), lay.t["R_codes"], R_sf, M, N, K, out_dtype=bf, ws=ws_g)
        Lu = X @ D
        Yu.add_(Lu @ U)
        # backward
        gc, gs, _ = ft.quantize_block16(dY)
        dXu, _ = ft.gemm_block16(gc, ft.mma_scales(gs, M, N), lay.t["R_codes_t"], R_sf_t, M, K, N, out_dtype=bf,
                                 ws=ws_g)
        P = dY @ U.t()
        dXu.add_(P @ D.t())
        dAu = X.t() @ P[:, r_sl]
        dBu = Lu[:, r_sl].t() @ dY
        return Yu, dXu, dAu, dBu

    # the 1x16 group-wise layout (§4.3, Table 5's comparator): Q16(R) and Q16(R^T)
    lay1 = ft.Linear1x16.from_weights(W, up(p["S_dn"]), up(p["S_up"]), A, B)
    wsf1, wsb1 = lay1.fwd_workspace(M), lay1.bwd_workspace(M)

    def w4a4g4_1x16():
        ft.linear_fwd_1x16(lay1, X, ws=wsf1, Y=Y, L=L)
        ft.linear_bwd_1x16(lay1, dY, X, L, ws=wsb1, dX=dX, dA=dA, dB=dB)

    fp4, lr = layer_work(M, K, N, r_s, r)
    out = {"workload": WORKLOAD, "steps": steps, "flop_per_step": fp4 + lr, "variants": {}}
    for name, fn in (("W4A4G4 1x16 groups + per-tensor scale", w4a4g4_1x16),
                     ("W4A16G4", w4a16g4), ("W4A4G16", w4a4g16), ("W4A16G16", w4a16g16),
                     ("bf16-LoRA ours (bf16 tensor cores)", lora_bf16_ours),
                     ("bf16-LoRA cuBLAS (torch.matmul)", lora_bf16_cublas),
                     ("W4A4G4 unfused (quantizer + 4-bit GEMM + cuBLAS low-rank)", unfused_w4)):
        for _ in range(warmup):
            flush.zero_()
            fn()
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for a, b in evs:
            flush.zero_()
            a.record()
            fn()
            b.record()
        torch.cuda.synchronize()
        ms = sum(a.elapsed_time(b) for a, b in evs) / steps
        out["variants"][name] = {"ms_per_step": ms, "tokens_per_s": M / (ms / 1e3),
                                 "tflops_equiv": (fp4 + lr) / (ms / 1e3) / 1e12}
    return out


def load_traffic(kernel):
    """DRAM bytes (read + write) per launch of `kernel` from the committed ncu
    summary profiles/traffic.txt; None when there is none or when the kernel's
    source file has changed since the counters were taken (git blob hash)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    try:
        with open(path) as f:
            for line in f:
                parts = line.split()
                if len(parts) != 4 or parts[0].startswith("#") or parts[0] != kernel:
                    continue
                with open(os.path.join(ROOT, parts[2]), "rb") as src:
                    data = src.read()
                blob = hashlib.sha1(b"blob %d\0" % len(data) + data).hexdigest()
                return int(parts[1]) if blob == parts[3] else None
    except Exception:
        return None
    return None


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="skip the other workloads' timings")
    ap.add_argument("--extra", default=",".join(EXTRA_WORKLOADS),
                    help="comma-separated subset of the other workloads to time (default: all)")
    ap.add_argument("--no-variants", action="store_true", help="skip the ablation variants' timings")
    args = ap.parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        return run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
