"""Benchmark: Falcon chunk-parallel forward, 8x12x2048x64 bf16 (chunk 64),
Falcon-1 and Falcon-1A, on one or more B200s (one process per GPU).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    torchrun --nproc-per-node N bench.py --gpus N ...

One step = one chunk-parallel forward of Falcon-1 and one of Falcon-1A over
the batch (B*L tokens each, all H heads), inputs resident in HBM.  L2 is
flushed (a 256 MiB write) before every timed step; each step is timed with
CUDA events on the launching stream and the job time is the max over ranks.
Each rank runs the full batch (weak scaling, no collective on the data path).

`--impl reference` times the fp64 CPU oracle (the only reference that exists
for this method) on a bounded sample of the same workload, on the host cores.
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

WORKLOAD = dict(name="falcon1-1A-chunk-bf16-8x12x2048x64", B=8, H=12, L=2048, dk=64, dv=64, chunk=64,
                variants=("F1", "F1A"), seed=20260002)
METRIC = "tokens/s for Falcon chunk-parallel fwd (H=12,d=64,L=2K) at 1 B200; % tensor/HBM peak"
DECODE = dict(variant="F2A", N=64, H=16, dk=128, dv=128, lam=0.02, seed=20260005)

# ncu summaries whose DRAM traffic the JSON line reports, with the sources the
# captured kernel was built from; a summary counts only while those sources
# hash to the value it records
CSRC = os.path.join(ROOT, "linear_attention_sequence_falcon_b200", "csrc")
PROFILED = {
    "chunk": ("chunk_local_kernel_falcon1_8x12x2048x64.md", ("k_chunk_split.cu", "tc_sm100.cuh", "common.cuh",
                                                               "params.h")),
    "decode": ("decode1_kernel_falcon2A_64x16x128x128.md", ("k_decode.cu", "common.cuh", "params.h")),
}
# GPU spin (cycles) queued before every timed step, so the host has enqueued
# the step's launches before its start event is reached
HEAD_START_CYCLES = 200_000


def source_hash(files):
    import hashlib
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(CSRC, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def profiled_traffic(key):
    """DRAM bytes per launch from the committed ncu summary, or None when the
    kernel's sources changed since the capture (or there is no summary)."""
    import re
    name, files = PROFILED[key]
    try:
        text = open(os.path.join(ROOT, "profiles", name)).read()
    except OSError:
        return None
    mh = re.search(r"source sha256: ([0-9a-f]{64})", text)
    mt = re.search(r"traffic per launch: (\d+) B", text)
    if not mh or not mt or mh.group(1) != source_hash(files):
        return None
    return int(mt.group(1))


def algorithmic_bytes_fwd(B, H, L, dk, dv, per_channel=False, elt=2):
    """Bytes a chunk-parallel forward must move at least once: q, k, v, beta
    and out in the input dtype plus the fp32 final state and lambda."""
    tok = B * H * L
    return tok * (2 * dk + dv + (dv if per_channel else 1) + dv) * elt + B * H * dv * dk * 4 + H * 4


# fp32 CUDA-core peak of a B200 at its maximum clock: 148 SMs x 128 FP32 lanes
# x 2 flop (one FMA) x 1965 MHz
FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def window_walk_flops(B, H, L, C, w, dv):
    """Flops of the chunk form's per-token solve for the C*B_w window errors
    of the regression family (Falcon-3), on the CUDA cores: token t of a
    chunk, window slot m and value channel j take the dot product of row
    t+m of the sample Gram with the per-row sums of the errors solved so far,
    which cover rows 0 .. t+B_w-2 (2 (t + B_w - 1) flops), plus 8 flops for
    the rest of the update.  Summed over full chunks."""
    per_chunk = dv * w * sum(2 * (t + w - 1) + 8 for t in range(C))
    return B * H * ((L + C - 1) // C) * per_chunk


def algorithmic_bytes_decode(N, H, dk, dv, per_channel=True, elt=2):
    """Per decode step: state read + write (fp32), x_prev read + write (fp32),
    q, k, v, beta in, out."""
    nh = N * H
    return nh * (2 * dv * dk * 4 + 2 * dk * 4 + (2 * dk + dv + (dv if per_channel else 1) + dv) * elt) + H * 4


class Clocks:
    """SM clock and throttle-reason sampler running during the timed region
    (NVML every 5 ms; the same counters nvidia-smi reports)."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4}

    def __init__(self, index):
        self.index = index
        self.rows = []
        self.stop = threading.Event()
        self.thread = None
        self.max_mhz = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            visible = os.environ.get("CUDA_VISIBLE_DEVICES")
            phys = int(visible.split(",")[self.index]) if visible else self.index
            self.h = pynvml.nvmlDeviceGetHandleByIndex(phys)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.thread = threading.Thread(target=self._run, daemon=True)
            self.thread.start()
            t0 = time.time()
            while not self.rows and time.time() - t0 < 2.0:
                time.sleep(0.005)
        except Exception:  # no NVML: leave the record empty
            self.thread = None
        return self

    def _run(self):
        nv = self.nv
        while not self.stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                    nv.nvmlDeviceGetCurrentClocksThrottleReasons
                rs = fn(self.h)
                self.rows.append((time.time(), mhz, rs))
            except Exception:
                pass
            time.sleep(0.005)

    def __exit__(self, *a):
        self.stop.set()
        if self.thread is not None:
            self.thread.join(timeout=2)

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"]}
        sm = [r[1] for r in self.rows]
        reasons = sorted({n for r in self.rows for n, bit in self.REASONS.items() if r[2] & bit})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(self.rows), "source": "nvml, 5 ms"}


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, 1590.0, "fallback"


def dist_setup(args):
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return rank, world, local


def _dist_device():
    import torch
    import torch.distributed as dist
    return "cuda" if dist.get_backend() == "nccl" else "cpu"


def max_over_ranks(x, world):
    """The job's time is the slowest rank's (one all-reduce MAX, no data-path collective)."""
    import torch
    import torch.distributed as dist
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=_dist_device())
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    import torch
    import torch.distributed as dist
    if world > 1:
        dist.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


def weak_scaling_value(world, tokens_per_step, steps, local_ms):
    """Whole-job tokens/s: every rank processes its own full batch (weak
    scaling), the job time is the max over ranks."""
    total_ms = max_over_ranks(local_ms, world)
    return world * tokens_per_step * steps / (total_ms / 1e3), total_ms


class OracleSample:
    """The fp64 oracle's chunk-parallel form on whole (b,h) units of the
    workload (Falcon-1 and Falcon-1A), one batch of units per call, on all
    host cores.  Inputs are drawn once, identical to the GPU run's."""

    def __init__(self):
        import oracle
        from linear_attention_sequence_falcon_b200 import inputs as gen
        w = WORKLOAD
        oracle.build()
        self.oracle = oracle
        self.d = gen.draw("F1", w["B"], w["H"], w["L"], w["dk"], w["dv"], seed=w["seed"], dtype="bf16")
        self.units = [(b, h) for b in range(w["B"]) for h in range(w["H"])]
        self.ncores = os.cpu_count() or 1
        self.next = 0
        self.threads = 1

    def step(self):
        """One batch of min(cores, units) units through both variants;
        returns (tokens, seconds)."""
        import numpy as np
        w = WORKLOAD
        n = min(self.ncores, len(self.units))
        batch = [self.units[(self.next + i) % len(self.units)] for i in range(n)]
        self.next = (self.next + n) % len(self.units)
        bs = [b for b, _ in batch]
        hs = [h for _, h in batch]
        # the selected units become the heads of one batch row, each with its own lambda
        sel = lambda a: np.ascontiguousarray(a[bs, hs][None])  # noqa: E731
        args = [sel(self.d[x]) for x in ("q_64", "k_64", "v_64", "beta_64")]
        lam = np.asarray(self.d["lam_64"])[hs]
        t0 = time.perf_counter()
        for variant in w["variants"]:
            _, _, self.threads = self.oracle.fwd(variant, "chunk", *args, lam, self.d["eps_64"], chunk=w["chunk"],
                                                 nthreads=self.ncores, return_threads=True)
        # a token is one position of one sequence with all H heads: n units are n/H of a sequence
        return len(w["variants"]) * n * w["L"] / w["H"], time.perf_counter() - t0


def cpu_oracle_sample(budget_s=12.0):
    """Oracle tokens/s over about budget_s of CPU wall time; returns
    (tokens/s, threads, units done, seconds)."""
    smp = OracleSample()
    tokens, used, units = 0, 0.0, 0
    while used < budget_s and units < len(smp.units):
        t, s = smp.step()
        tokens += t
        used += s
        units += min(smp.ncores, len(smp.units))
    return tokens / used, smp.threads, units, used


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    smp = OracleSample()
    for _ in range(args.warmup):
        smp.step()
    tokens, used = 0, 0.0
    for _ in range(args.steps):
        t, s = smp.step()
        tokens += t
        used += s
    value = tokens / used
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": used / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": smp.threads, "kind": "oracle",
                             "sample": "each step: %d whole (b,h) units of the workload through the fp64 oracle's "
                                       "chunk-parallel form, Falcon-1 and Falcon-1A; H units make one token of "
                                       "the metric" % min(smp.ncores, len(smp.units))},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def workload_config():
    w = WORKLOAD
    return {"workload": w["name"], "B": w["B"], "H": w["H"], "L": w["L"], "d_k": w["dk"], "d_v": w["dv"],
            "chunk": w["chunk"], "variants": list(w["variants"]), "global_batch": w["B"], "seq_len": w["L"],
            "l2": "flushed (256 MiB write) before every timed step", "parallelism": "replicas"}


def run_ours(args):
    import torch
    import linear_attention_sequence_falcon_b200 as F
    from linear_attention_sequence_falcon_b200 import build, inputs as gen
    build.build()
    F.load()
    rank, world, local = dist_setup(args)
    w = WORKLOAD
    d = gen.draw("F1", w["B"], w["H"], w["L"], w["dk"], w["dv"], seed=w["seed"] + 1000 * rank, dtype="bf16")
    q, k, v, beta, lam = (d[n].cuda() for n in ("q", "k", "v", "beta", "lam"))
    outs = {var: torch.empty((w["B"], w["H"], w["L"], w["dv"]), dtype=torch.bfloat16, device="cuda")
            for var in w["variants"]}
    states = {var: torch.empty((w["B"], w["H"], w["dv"], w["dk"]), dtype=torch.float32, device="cuda")
              for var in w["variants"]}
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    # the caller-owned workspace of each forward (falcon_fwd_ws), allocated
    # once: no stream-ordered allocation runs inside the timed region
    ws = {var: torch.empty(F.fwd_workspace_size(var, "chunk", torch.bfloat16, w["B"], w["H"], w["L"], w["dk"],
                                                w["dv"], chunk=w["chunk"]), dtype=torch.uint8, device="cuda")
          for var in w["variants"]}

    def step(ev=None):
        for var in w["variants"]:
            if ev is not None:
                ev[var][0].record(stream)
            F.fwd(var, "chunk", q, k, v, beta, lam, d["eps"], chunk=w["chunk"], out=outs[var],
                  final_state=states[var], stream=stream, workspace=ws[var])
            if ev is not None:
                ev[var][1].record(stream)

    if args.profile:
        # device step only, for profilers (which flush caches themselves)
        for _ in range(args.warmup + args.steps):
            step()
        torch.cuda.synchronize()
        return
    if args.profile_decode:
        args.steps = max(args.steps, 1)
        wdw = args.decode_window
        measure_decode(F, gen, stream, flush, peaks()[0], args, profile=True,
                       variant="F3" if wdw > 1 else None, window=wdw)
        return
    for _ in range(max(args.warmup, 3)):
        flush.zero_()
        step()
    barrier(world)
    # blocks that gave up on a bounded wait leave incomplete outputs while the
    # call returns OK: the counter must not move over the measured steps
    timeouts_before = F.wait_timeouts()
    per_var = {var: [] for var in w["variants"]}
    step_ms = []
    with Clocks(local) as clk:
        for _ in range(args.steps):
            flush.zero_()
            torch.cuda._sleep(HEAD_START_CYCLES)
            ev = {var: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for var in w["variants"]}
            step(ev)
            torch.cuda.synchronize()
            for var in w["variants"]:
                per_var[var].append(ev[var][0].elapsed_time(ev[var][1]))
            step_ms.append(sum(ev[var][0].elapsed_time(ev[var][1]) for var in w["variants"]))
        barrier(world)
    tokens_per_step = len(w["variants"]) * w["B"] * w["L"]
    value, total_ms = weak_scaling_value(world, tokens_per_step, args.steps, sum(step_ms))

    # end to end through the C ABI on pinned host buffers: falcon_fwd_host
    # copies the inputs in, runs both variants and copies outputs and states
    # back, the batch cut into slices so that copies and compute overlap
    hq, hk, hv, hb, hl = (d[n].pin_memory() for n in ("q", "k", "v", "beta", "lam"))
    ho = [torch.empty_like(outs[var], device="cpu").pin_memory() for var in w["variants"]]
    hs = [torch.empty_like(states[var], device="cpu").pin_memory() for var in w["variants"]]
    e2e_ms = []
    for i in range(max(args.warmup, 3) + args.steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        F.fwd_host(w["variants"], "chunk", hq, hk, hv, hb, hl, d["eps"], chunk=w["chunk"], out=ho,
                   final_state=hs, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize()
        if i >= max(args.warmup, 3):
            e2e_ms.append(e0.elapsed_time(e1))
    e2e_value, _ = weak_scaling_value(world, tokens_per_step, args.steps, sum(e2e_ms))
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hb, hl))
    d2h = sum(t.numel() * t.element_size() for t in ho + hs)

    hbm, tflops, src = peaks()
    f1_ms = statistics.mean(per_var["F1"])
    ab = algorithmic_bytes_fwd(w["B"], w["H"], w["L"], w["dk"], w["dv"])
    achieved = ab / (f1_ms / 1e3) / 1e9
    roof = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
            "traffic": profiled_traffic("chunk"),
            "kernel": "one Falcon-1 chunk-parallel forward (chunk_local_kernel + chunk_chain_kernel)",
            "peak_source": src,
            "algorithmic_bytes_per_launch": ab, "launch_ms": f1_ms}

    decode = measure_decode(F, gen, stream, flush, hbm, args) if not args.no_decode else None
    timeouts_delta = int(max_over_ranks(float(F.wait_timeouts() - timeouts_before), world))
    if timeouts_delta != 0:
        print(json.dumps({"metric": METRIC, "error": "%d tensor-core thread blocks gave up on a bounded wait "
                          "during the measured steps: outputs incomplete, no value reported" % timeouts_delta}),
              flush=True)
        sys.exit(3)

    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": workload_config(), "roofline": roof,
            "per_variant_ms": {var: statistics.mean(per_var[var]) for var in w["variants"]},
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            # every falcon_fwd of this shape is two kernels: chunk_local_kernel + chunk_chain_kernel
            "gpu_launches": 2 * len(w["variants"]) * args.steps, "clocks": clk.summary(),
            "wait_timeouts_delta": timeouts_delta}
    if decode is not None:
        line["decode"] = decode
        # the window path (Falcon-3, window 4) and d = 64 decode, same batch and heads
        line["decode_more"] = [measure_decode(F, gen, stream, flush, hbm, args, variant="F3", window=4),
                               measure_decode(F, gen, stream, flush, hbm, args, variant="F1", dk=64)]
    if not args.no_extras:
        # the chunk-length sweep and the backward on the same workload (extra keys, not the headline)
        line["chunk_sweep"] = chunk_sweep_rows(F, gen, flush, args.steps)
        line["backward"] = backward_rows(F, gen, flush, args.steps)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tps, threads, units, used = cpu_oracle_sample(budget_s=args.cpu_budget)
        line["cpu_baseline"] = {"value": tps, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                                "sample": "fp64 oracle chunk-parallel form, Falcon-1 and Falcon-1A, %d whole (b,h) "
                                          "units of the workload (%.1f s); H units make one token of the "
                                          "metric" % (units, used)}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def measure_decode(F, gen, stream, flush, hbm, args, profile=False, variant=None, dk=None, window=1):
    """Decode row: one falcon_decode_step per step for N sequences (by
    default Falcon-2A, N=64, H=16, 128x128 fp32 state per head, 64 MiB of
    state).  Steps rotate over four independent sets of states and carries
    (256 MiB in all at d = 128, twice L2), so no step finds its state in L2;
    the dirty lines a step leaves are written back during later steps, as in
    steady-state serving."""
    import torch
    dd = DECODE
    variant = variant or dd["variant"]
    N, H = dd["N"], dd["H"]
    dk = dv = dk or dd["dk"]
    pool = 16
    sets = 4 if dk == 128 else 16  # at least twice L2 of states in rotation
    d = gen.draw_decode(variant, N, H, dk, dv, pool, seed=dd["seed"], lam=dd["lam"])
    q, k, v, beta = (d[n].cuda() for n in ("q", "k", "v", "beta"))
    lam = d["lam"].cuda()
    state = [torch.zeros((N, H, dv, dk), dtype=torch.float32, device="cuda") for _ in range(sets)]
    x_prev = [torch.zeros((N, H, dk), dtype=torch.float32, device="cuda") for _ in range(sets)]
    win = [torch.zeros((N, H, window - 1, dk + dv), dtype=torch.float32, device="cuda") if window > 1 else None
           for _ in range(sets)]
    out = torch.empty((N, H, dv), dtype=torch.bfloat16, device="cuda")
    steps = max(args.steps, 20)

    def one(i):
        F.decode_step(variant, q[i % pool], k[i % pool], v[i % pool], beta[i % pool], lam, d["eps"], window,
                      state[i % sets], x_prev[i % sets], win[i % sets], out=out, stream=stream)

    if profile:  # decode steps only, for profilers
        for i in range(args.warmup + args.steps):
            one(i)
        torch.cuda.synchronize()
        return None
    for i in range(max(args.warmup, 3) * sets):
        one(i)
    ms = []
    for i in range(steps):
        torch.cuda._sleep(HEAD_START_CYCLES)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        one(i)
        e1.record(stream)
        torch.cuda.synchronize()
        ms.append(e0.elapsed_time(e1))
    t = statistics.mean(ms)
    per_channel = variant in ("F2", "F2A")
    ab = algorithmic_bytes_decode(N, H, dk, dv, per_channel=per_channel)
    if window > 1:  # the window carry is read and written too
        ab += N * H * (window - 1) * (dk + dv) * 4 * 2
    gbs = ab / (t / 1e3) / 1e9
    # the kernel the library picks for this shape
    if window == 1:
        kernel = "decode1r_kernel" if dk == 64 and dv <= 64 else "decode1_kernel"
    else:
        kernel = "decodew_kernel" if window <= 4 else "decode_kernel"
    return {"workload": "%s-decode-bf16-N%dxH%d-state%dx%d-fp32%s" % (
                variant.replace("F", "falcon"), N, H, dv, dk, "-window%d" % window if window > 1 else ""),
            "kernel": kernel, "us_per_step": t * 1e3, "tokens_per_s": N / (t / 1e3), "steps": steps,
            "l2": "%d rotating sets of states and carries (%d MiB, over 2x L2); no flush"
                  % (sets, sets * N * H * dv * dk * 4 >> 20),
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                         "algorithmic_bytes_per_launch": ab,
                         "traffic": profiled_traffic("decode") if (variant, dk, window) == (dd["variant"], 128, 1)
                         else None}}


def time_call(fn, flush, steps, stream=None):
    """Median CUDA-event time (ms) of fn() over `steps` calls (3..20), L2
    flushed and a GPU head start queued before each, after one warm-up call."""
    import torch
    fn()
    torch.cuda.synchronize()
    ms = []
    for _ in range(max(3, min(steps, 20))):
        flush.zero_()
        torch.cuda._sleep(HEAD_START_CYCLES)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        torch.cuda.synchronize()
        ms.append(e0.elapsed_time(e1))
    return statistics.median(ms)


SWEEP_KERNELS = {16: "seq_chunk_kernel<16>", 32: "seq_chunk_kernel<32>", 64: "chunk_local_kernel + chunk_chain_kernel",
                 128: "seq_chunk_kernel<128>"}


def chunk_sweep_rows(F, gen, flush, steps):
    """The chunk-parallel forward of workload 2 (Falcon-1 and Falcon-1A,
    8x12x2048x64 bf16) at chunk 16, 32, 64 and 128 under the prefix pair and
    at 64 under the same-step pair; every point on the tensor cores."""
    import torch
    w = gen.WORKLOADS[2]
    rows = []
    for var in w["variants"]:
        d = gen.workload_inputs(2, var)
        a = [d[k].cuda() for k in ("q", "k", "v", "beta", "lam")]
        out = torch.empty((w["B"], w["H"], w["L"], w["dv"]), dtype=torch.bfloat16, device="cuda")
        S = torch.empty((w["B"], w["H"], w["dv"], w["dk"]), dtype=torch.float32, device="cuda")
        for chunk, pairing in ((16, "prefix"), (32, "prefix"), (64, "prefix"), (128, "prefix"), (64, "same_step")):
            need = F.fwd_workspace_size(var, "chunk", torch.bfloat16, w["B"], w["H"], w["L"], w["dk"], w["dv"],
                                        chunk=chunk, pairing=pairing)
            ws = torch.empty(max(need, 1), dtype=torch.uint8, device="cuda")
            t = time_call(lambda: F.fwd(var, "chunk", *a, d["eps"], chunk=chunk, pairing=pairing, out=out,
                                        final_state=S, workspace=ws), flush, steps)
            rows.append({"variant": var, "chunk": chunk, "pairing": pairing, "ms": t,
                         "tokens_per_s": w["B"] * w["L"] / (t / 1e3), "kernels": SWEEP_KERNELS[chunk],
                         "workspace_bytes": need})
    return rows


def backward_rows(F, gen, flush, steps, variants=("F1", "F1A"), forms=("chunk", "recurrent")):
    """falcon_bwd_ex on workload 2 (8x12x2048x64 bf16): the chunk-parallel
    backward and the recurrent one, each against the algorithmic bytes
    (q, k, v, beta, dout read in bf16; dq, dk, dv, dbeta written in fp32)."""
    import numpy as np
    import torch
    w = gen.WORKLOADS[2]
    B, H, L, dk, dv = w["B"], w["H"], w["L"], w["dk"], w["dv"]
    hbm, _, src = peaks()
    rng = np.random.default_rng(20260102)
    do = torch.from_numpy(rng.standard_normal((B, H, L, dv)).astype(np.float32)).to(torch.bfloat16).cuda()
    ds = torch.from_numpy(rng.standard_normal((B, H, dv, dk)).astype(np.float32)).cuda()
    tok = B * H * L
    ab = tok * (dk + dk + dv + 1 + dv) * 2 + tok * (dk + dk + dv + 1) * 4 + B * H * dv * dk * 4
    out = {}
    for var in variants:
        d = gen.workload_inputs(2, var)
        a = [d[k].cuda() for k in ("q", "k", "v", "beta", "lam")]
        for form in forms:
            t = time_call(lambda: F.bwd(var, *a, d["eps"], do, ds, form=form), flush, steps)
            gbs = ab / (t / 1e3) / 1e9
            out["%s_%s" % (var, form)] = {"ms": t, "tokens_per_s": B * L / (t / 1e3),
                                          "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s",
                                                       "frac": gbs / hbm, "peak_source": src,
                                                       "algorithmic_bytes_per_launch": ab}}
    return out


def run_workloads(args):
    """--workloads: one JSON line per (workload, variant, form) of the
    workloads table (inputs.WORKLOADS): CUDA events around one falcon_fwd,
    after a warm-up call, L2 flushed before each timed call; median of
    --steps calls (at least 3, at most 20).  Not the contract line."""
    import torch
    import linear_attention_sequence_falcon_b200 as F
    from linear_attention_sequence_falcon_b200 import build, inputs as gen
    build.build()
    F.load()
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")
    cases = []
    for n, w in gen.WORKLOADS.items():
        if args.only and n != args.only:
            continue
        forms = list(w["forms"])
        if n in (2, 4):  # the parallel forms beside the recurrent kernel on the same inputs
            forms = ["chunk", "masked", "recurrent"]
        for var in w["variants"]:
            for form in forms:
                cases.append((n, w, var, form))
    for n, w, var, form in cases:
        d = gen.workload_inputs(n, var)
        args_ = [d[k].cuda() for k in ("q", "k", "v", "beta", "lam")]
        out, S = F.fwd(var, form, *args_, d["eps"], window=w["window"], chunk=w["chunk"])
        torch.cuda.synchronize()
        ms = []
        for _ in range(max(3, min(args.steps, 20))):
            flush.zero_()
            torch.cuda._sleep(HEAD_START_CYCLES)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            F.fwd(var, form, *args_, d["eps"], window=w["window"], chunk=w["chunk"], out=out, final_state=S)
            e1.record()
            torch.cuda.synchronize()
            ms.append(e0.elapsed_time(e1))
        t = statistics.median(ms)
        elt = 2 if w["dtype"] == "bf16" else 4
        ab = algorithmic_bytes_fwd(w["B"], w["H"], w["L"], w["dk"], w["dv"], per_channel=var in ("F2", "F2A"),
                                   elt=elt)
        gbs = ab / (t / 1e3) / 1e9
        hbm, _, peak_src = peaks()
        line = {"workload": n, "name": w["name"], "variant": var, "form": form, "dtype": w["dtype"],
                "ms": t, "tokens_per_s": w["B"] * w["L"] / (t / 1e3),
                "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                             "peak_source": peak_src, "algorithmic_bytes_per_launch": ab}}
        if form == "chunk" and var == "F3":
            # the per-token window solve runs on the CUDA cores: its fp32 roofline
            fl = window_walk_flops(w["B"], w["H"], w["L"], w["chunk"], w["window"], w["dv"])
            tfs = fl / (t / 1e3) / 1e12
            line["roofline_alu"] = {"bound": "alu", "achieved": tfs, "peak": FP32_ALU_TFLOPS, "unit": "TFLOP/s",
                                    "frac": tfs / FP32_ALU_TFLOPS, "flops_per_launch": fl,
                                    "peak_source": "148 SMs x 128 FP32 lanes x 2 x 1965 MHz"}
        if not args.no_cpu_baseline:
            line["cpu_oracle"] = workload_oracle_rate(d, var, form, w)
        print(json.dumps(line), flush=True)


def run_chunk_sweep(args):
    """--chunk-sweep: chunk_sweep_rows as one JSON line each.  Not the contract line."""
    import torch
    import linear_attention_sequence_falcon_b200 as F
    from linear_attention_sequence_falcon_b200 import build, inputs as gen
    build.build()
    F.load()
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")
    for row in chunk_sweep_rows(F, gen, flush, args.steps):
        print(json.dumps(dict(sweep="chunk", workload=gen.WORKLOADS[2]["name"], **row)), flush=True)


def run_backward(args):
    """--backward: falcon_bwd on workload 2 (Falcon-1 and Falcon-1A,
    8x12x2048x64 bf16), workload 3 (Falcon-2, 4x16x4096x128), workload 4
    (Falcon-3 and Falcon-3A, window 4) and workload 5's prefill (Falcon-2A,
    2x16x32768x128 bf16): CUDA events around one call after a
    warm-up call, L2 flushed, median of --steps calls (3..10); an HBM
    roofline on the algorithmic bytes (q, k, v, beta, dout read; dq, dk, dv,
    dbeta written in fp32) and the fp64 oracle's reverse mode on whole (b,h)
    units (workloads 2 and 4: its state history at L = 32768, d = 128 would
    take 4 GB per unit).  Not the contract line."""
    import numpy as np
    import torch
    import linear_attention_sequence_falcon_b200 as F
    from linear_attention_sequence_falcon_b200 import build, inputs as gen
    build.build()
    F.load()
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")
    hbm, _, peak_src = peaks()
    for n, var in ((2, "F1"), (2, "F1A"), (3, "F2"), (4, "F3"), (4, "F3A"), (5, "F2A")):
        if args.only and n != args.only:
            continue
        if args.bwd_form == "chunk" and var not in ("F1", "F1A"):
            continue  # the chunk-parallel backward covers Falcon-1/1A (bf16, d = 64)
        w = gen.WORKLOADS[n]
        d = gen.workload_inputs(n, var)
        B, H, L, dk, dv = w["B"], w["H"], w["L"], w["dk"], w["dv"]
        rng = np.random.default_rng(20260100 + n)
        do = torch.from_numpy(rng.standard_normal((B, H, L, dv)).astype(np.float32)).to(torch.bfloat16).cuda()
        ds = torch.from_numpy(rng.standard_normal((B, H, dv, dk)).astype(np.float32)).cuda()
        a = [d[k].cuda() for k in ("q", "k", "v", "beta", "lam")]
        F.bwd(var, *a, d["eps"], do, ds, window=w["window"], form=args.bwd_form)
        torch.cuda.synchronize()
        ms = []
        for _ in range(max(3, min(args.steps, 10))):
            flush.zero_()
            torch.cuda._sleep(HEAD_START_CYCLES)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            F.bwd(var, *a, d["eps"], do, ds, window=w["window"], form=args.bwd_form)
            e1.record()
            torch.cuda.synchronize()
            ms.append(e0.elapsed_time(e1))
        t = statistics.median(ms)
        nb = dv if var in ("F2", "F2A") else 1
        tok = B * H * L
        ab = tok * (dk + dk + dv + nb + dv) * 2 + tok * (dk + dk + dv + nb) * 4 + B * H * dv * dk * 4
        gbs = ab / (t / 1e3) / 1e9
        kern = ("chunk_local_kernel + chunk_chain_kernel + bwd_rchain_kernel + bwd_chunk_kernel"
                if args.bwd_form == "chunk" else
                "bwd_prep_kernel + bwd_sweep_kernel + bwd_decay_kernel + bwd_key_kernel")
        line = {"backward": var, "form": args.bwd_form, "workload": w["name"], "ms": t,
                "tokens_per_s": B * L / (t / 1e3), "kernels": kern,
                "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                             "peak_source": peak_src, "algorithmic_bytes_per_launch": ab}}
        if n in (2, 4) and not args.no_cpu_baseline:
            import oracle
            oracle.build()
            units = [(b, h) for b in range(B) for h in range(H)][:min(os.cpu_count() or 1, B * H)]
            bs, hs = [u[0] for u in units], [u[1] for u in units]
            sel = lambda x: np.ascontiguousarray(x[bs, hs][None])  # noqa: E731
            t0 = time.perf_counter()
            oracle.bwd(var, *(sel(d[k]) for k in ("q_64", "k_64", "v_64", "beta_64")), np.asarray(d["lam_64"])[hs],
                       d["eps_64"], sel(do.double().cpu().numpy()), sel(ds.double().cpu().numpy()), window=w["window"])
            sec = time.perf_counter() - t0
            line["cpu_oracle"] = {"value": len(units) * L / H / sec, "unit": "tokens/s", "cores": os.cpu_count(),
                                  "kind": "oracle", "sample": "fp64 reverse mode, %d whole (b,h) units, %.1f s"
                                  % (len(units), sec)}
        print(json.dumps(line), flush=True)


def workload_oracle_rate(d, variant, form, w):
    """The fp64 oracle in the row's own form -- the recurrent form for masked
    rows, whose O(L^2) oracle takes 7-80 s per (b,h) unit at L = 2048 -- on
    min(cores, B*H) whole (b,h) units of the workload's inputs, all host
    cores: tokens/s."""
    import numpy as np
    import oracle
    oracle.build()
    units = [(b, h) for b in range(w["B"]) for h in range(w["H"])]
    n = min(os.cpu_count() or 1, len(units))
    bs = [b for b, _ in units[:n]]
    hs = [h for _, h in units[:n]]
    sel = lambda a: np.ascontiguousarray(a[bs, hs][None])  # noqa: E731
    args = [sel(d[x]) for x in ("q_64", "k_64", "v_64", "beta_64")]
    lam = np.asarray(d["lam_64"])[hs]
    oform = "recurrent" if form == "masked" else form
    reps, sec = 0, 0.0
    while sec < 1.0 and reps < 100:  # repeated to about a second of wall time
        t0 = time.perf_counter()
        _, _, threads = oracle.fwd(variant, oform, *args, lam, d["eps_64"], window=w["window"],
                                   chunk=w["chunk"], nthreads=os.cpu_count() or 1, return_threads=True)
        sec += time.perf_counter() - t0
        reps += 1
    # a token is one position of one sequence with all H heads
    return {"value": reps * n * w["L"] / w["H"] / sec, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": "fp64 %s form, %d whole (b,h) units x %d runs, %.2f s" % (oform, n, reps, sec)}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-extras", action="store_true", help="leave out the chunk sweep and backward keys")
    ap.add_argument("--profile-decode", action="store_true",
                    help="run only warmup+steps decode steps (no flush or JSON), for ncu")
    ap.add_argument("--decode-window", type=int, default=1,
                    help="with --profile-decode: the Falcon-3 window decode of this window (2-8) instead")
    ap.add_argument("--workloads", action="store_true",
                    help="time every workload and form of the workloads table, one JSON line each")
    ap.add_argument("--only", type=int, default=0, help="with --workloads or --backward: just this workload number")
    ap.add_argument("--backward", action="store_true",
                    help="time falcon_bwd on workloads 2 (Falcon-1, -1A), 3 (Falcon-2) and 5's prefill (Falcon-2A)")
    ap.add_argument("--bwd-form", default="recurrent", choices=["recurrent", "chunk"],
                    help="with --backward: the form whose derivative is taken")
    ap.add_argument("--chunk-sweep", action="store_true",
                    help="the chunk form of workload 2 at chunk 16/32/64 and both pairings (one line each)")
    ap.add_argument("--profile", action="store_true",
                    help="run only warmup+steps device steps (no flush, e2e, clocks or JSON), for ncu")
    args = ap.parse_args()
    if args.chunk_sweep:
        return run_chunk_sweep(args)
    if args.backward:
        return run_backward(args)
    if args.workloads:
        run_workloads(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
