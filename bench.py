#!/usr/bin/env python
"""Benchmark of the DSA prefill chunk (indexer -> exact top-k -> sparse MLA) on B200.

One step = one dsa_prefill_chunk call over one synthetic chunk resident in HBM
(default: the 128K-context workload, N = 131,072 cached keys, L = 1,024
queries).  Prints one JSON line on rank 0.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

With --gpus N > 1 and no torch.distributed environment (RANK / WORLD_SIZE
unset), bench.py starts the N ranks itself under torch.distributed.run on this
node (127.0.0.1) and passes its exit status on.

Timing: W untimed warm-up steps; then K steps, each preceded by a 512 MiB
device write that flushes the 126 MB L2, each bracketed by CUDA events on the
launching stream (the flush is outside the events); a barrier and a device
synchronise on both sides of the timed region; max over ranks.  nvidia-smi
samples clocks and throttle reasons from 0.4 s of untimed steps before the
timed region until 0.4 s after it, so the record is taken under load.  With N > 1
every rank runs an independent replica (the path has no cross-GPU exchange):
value = all ranks' query tokens / max rank time (weak scaling).

--impl reference times the CPU oracle (the plain fp64 C implementation the
tests compare against) on the host cores, on a bounded sample of the same
workload's queries.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

import dsa_inputs  # noqa: E402

METRIC = "DSA prefill query tokens/s at 128K ctx (indexer+top-k+sparse MLA); % roofline"
UNIT = "tokens/s"
L2_FLUSH_BYTES = 512 << 20
LOAD_WINDOW_S = 0.4  # untimed steps on each side of the timed region while the clocks are sampled
EVENTS_PER_BLOCK = 7


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def measured_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def indexer_kernel_traffic(cfg) -> int | None:
    """DRAM bytes per launch of the main indexer kernel from the committed ncu summary, if it still applies."""
    path = os.path.join(ROOT, "profiles", "indexer_main_traffic.txt")
    src = os.path.join(ROOT, "deepseek_sparse_attention_relu_b200", "csrc", "indexer.cu")
    if not os.path.exists(path):
        return None
    with open(src, "rb") as f:
        sha = hashlib.sha256(f.read()).hexdigest()[:16]
    vals = {}
    with open(path) as f:
        for line in f:
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                vals[k.strip()] = v.strip()
    if vals.get("indexer_cu_sha256_16") != sha or vals.get("workload") != cfg.name:
        return None
    try:
        return int(float(vals["dram_bytes_per_launch"]))
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples (every 200 ms) while the GPU runs the timed region and the
    untimed load window around it."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.05)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def keep_busy(step_fn, seconds: float, sync) -> int:
    """Run untimed steps back to back for about `seconds` of wall time (at least one), then wait for the
    device.  Used around the timed region so that the clock sampler sees the GPU under load: the timed
    region itself is often shorter than one sampling interval."""
    n = 0
    t0 = time.perf_counter()
    while True:
        step_fn()
        n += 1
        if n % 8 == 0:
            sync()
            if time.perf_counter() - t0 >= seconds:
                break
    sync()
    return n


def max_over_ranks(value: float, world: int, device=None) -> float:
    """The largest value over all ranks (every rank must call it; identity when world == 1).

    Times of a multi-GPU run are taken as the slowest rank's, so the job's
    throughput is all ranks' work divided by that time.
    """
    if world <= 1:
        return float(value)
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank: int, world: int, steps: int, max_total_ms: float) -> float:
    """Whole-job query tokens per second: every rank runs its own replica of the chunk."""
    return world * tokens_per_rank * steps / (max_total_ms / 1000.0)


def spawn_ranks(gpus: int, argv: list[str]) -> int:
    """Re-run this script as `gpus` ranks under torch.distributed.run on this node; returns the exit status."""
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={gpus}",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__), *argv]
    log(f"[bench] starting {gpus} ranks: {' '.join(cmd)}")
    return subprocess.call(cmd)


def measure_fp8_peak(dev, n: int = 8192, reps: int = 10) -> float | None:
    """Dense e4m3 tensor throughput on this GPU (TFLOP/s): torch._scaled_mm of two n x n e4m3 matrices with
    bf16 output, best of `reps` CUDA-event-timed calls (2 n^3 flops each).  None if the call is unavailable."""
    try:
        g = torch.Generator(device=dev).manual_seed(7)
        a = torch.randn(n, n, device=dev, generator=g).to(torch.float8_e4m3fn)
        b = torch.randn(n, n, device=dev, generator=g).to(torch.float8_e4m3fn)
        one = torch.ones((), device=dev, dtype=torch.float32)
        run = lambda: torch._scaled_mm(a, b.t(), scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        for _ in range(3):
            run()
        best = float("inf")
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            run()
            e1.record()
            torch.cuda.synchronize()
            best = min(best, e0.elapsed_time(e1))
        del a, b
        return 2.0 * n ** 3 / (best / 1000.0) / 1e12
    except (RuntimeError, TypeError) as e:
        log(f"[bench] fp8 peak not measured: {e}")
        return None


def run_dry(args, rank: int, world: int) -> None:
    """The launch and cross-rank plumbing alone, on CPU ranks (gloo): every rank 'times' a fixed sleep per step,
    the slowest rank's total is taken, rank 0 prints the JSON line.  Used by the CPU tests of the launcher."""
    import torch.distributed as dist
    if world > 1:
        dist.init_process_group("gloo")
    cfg = dsa_inputs.BY_NAME[args.workload]
    per_step_s = 0.001 * (1 + rank)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        time.sleep(per_step_s)
    total_ms = max_over_ranks((time.perf_counter() - t0) * 1000.0, world)
    if rank == 0:
        print(json.dumps({"dry_run": True, "metric": METRIC, "n_gpus": world, "steps": args.steps,
                          "ms_per_step": total_ms / args.steps,
                          "value": job_throughput(cfg.L, world, args.steps, total_ms), "unit": UNIT}), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def cpu_oracle_rate(cfg, inp, rows: list[int], threads: int) -> tuple[float, float]:
    """Query tokens/s of the unmodified oracle over `rows` on `threads` host threads; returns (rate, seconds)."""
    import oracle
    pb = oracle.Problem(dsa_inputs.raw_bits(inp["q_idx"]), dsa_inputs.raw_bits(inp["k_idx"]), inp["w"],
                        cfg.idx_code, cfg.L, cfg.N, cfg.H_I, cfg.D_I, cfg.q_pos0, cfg.topk,
                        q=dsa_inputs.raw_bits(inp["q"]), kv=dsa_inputs.raw_bits(inp["kv"]), H=cfg.H, scale=cfg.scale)
    t0 = time.perf_counter()
    oracle.map_rows(lambda t: oracle.prefill_row(pb, t), rows, threads=threads)
    dt = time.perf_counter() - t0
    return len(rows) / dt, dt


def sample_rows(cfg, n: int, salt: int = 0) -> list[int]:
    g = torch.Generator().manual_seed(1234 + salt)
    return sorted(torch.randperm(cfg.L, generator=g)[:min(n, cfg.L)].tolist())


def flops_and_bytes(cfg) -> dict:
    pairs = cfg.visible_pairs()
    idx_flop = pairs * 2 * cfg.H_I * cfg.D_I
    mla_flop = cfg.L * cfg.H * cfg.topk * (576 + 512) * 2
    esz = 1 if cfg.idx_dtype == "e4m3" else 2
    alg_bytes = (cfg.N * cfg.D_I * esz + cfg.L * cfg.H_I * cfg.D_I * esz + cfg.L * cfg.H_I * 4
                 + min(cfg.N, cfg.L * cfg.topk) * 1152 + cfg.L * cfg.H * 576 * 2 + cfg.L * cfg.H * 512 * 2
                 + cfg.L * cfg.topk * 4)
    return {"pairs": pairs, "indexer_flop": idx_flop, "mla_flop": mla_flop, "alg_bytes": alg_bytes}


def run_reference(args, rank: int, world: int) -> None:
    if rank != 0:
        return
    cfg = dsa_inputs.BY_NAME[args.workload]
    inp = dsa_inputs.generate(cfg)
    threads = os.cpu_count() or 1
    rows_per_step = max(1, min(cfg.L, threads))
    for w in range(args.warmup):
        cpu_oracle_rate(cfg, inp, sample_rows(cfg, max(1, rows_per_step // 4), salt=100 + w), threads)
    total_rows, total_s = 0, 0.0
    for k in range(args.steps):
        rows = sample_rows(cfg, rows_per_step, salt=k)
        _, dt = cpu_oracle_rate(cfg, inp, rows, threads)
        total_rows += len(rows)
        total_s += dt
    value = total_rows / total_s
    sample = (f"{args.steps} steps x {rows_per_step} seeded-random query rows of the workload "
              f"(full indexer row + exact top-k + attention per row)")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * total_s / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": cfg.name, "N": cfg.N, "L": cfg.L, "topk": cfg.topk, "H": cfg.H, "H_I": cfg.H_I,
                   "D_I": cfg.D_I, "indexer_dtype": cfg.idx_dtype, "parallelism": "replicas"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }), flush=True)


def run_ours(args, rank: int, world: int, local_rank: int) -> None:
    import deepseek_sparse_attention_relu_b200 as dsa

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    cfg = dsa_inputs.BY_NAME[args.workload]
    t_gen = time.perf_counter()
    inp = dsa_inputs.generate(cfg)
    log(f"[bench] rank {rank}: generated {cfg.name} in {time.perf_counter() - t_gen:.1f}s")
    g = {k: v.to(dev) for k, v in inp.items()}
    out = torch.empty(cfg.L, cfg.H, 512, dtype=torch.bfloat16, device=dev)
    dt = dsa.DSA_BF16 if cfg.idx_dtype == "bf16" else dsa.DSA_FP8_E4M3
    ws = dsa.alloc_workspace(dsa.dsa_prefill_chunk_workspace(cfg.L, cfg.N, cfg.H_I, cfg.D_I, cfg.H, cfg.topk, 0, dt,
                                                             False), dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    nblocks = (cfg.L + 1023) // 1024
    stream = torch.cuda.current_stream()

    def new_events(n):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        for e in evs:
            e.record(stream)  # materialise the handle
        return evs

    def step(events):
        dsa.dsa_prefill_chunk_profiled(g["q_idx"], g["k_idx"], g["w"], g["q"], g["kv"], cfg.q_pos0, cfg.topk,
                                       cfg.scale, out, events, workspace=ws)

    warm_ev = new_events(EVENTS_PER_BLOCK * nblocks)
    for _ in range(args.warmup):
        flush.zero_()
        step(warm_ev)
    torch.cuda.synchronize()
    status = dsa.dsa_workspace_status(ws)
    if status != 0:
        raise RuntimeError(f"device status word {status:#x} after warm-up")

    starts = new_events(args.steps)
    ends = new_events(args.steps)
    # Timed steps record only the two events that bracket each block's main
    # indexer pass (its live duration for the roofline): every event between two
    # kernels also stops the next one from launching early (programmatic
    # dependent launch), so the other stage boundaries are left unmarked here
    # and the stage breakdown comes from separate untimed steps below.
    main_ev = [new_events(2 * nblocks) for _ in range(args.steps)]

    def timed_events(k):
        evs = [None] * (EVENTS_PER_BLOCK * nblocks)
        for b in range(nblocks):
            evs[EVENTS_PER_BLOCK * b + 2] = main_ev[k][2 * b]
            evs[EVENTS_PER_BLOCK * b + 3] = main_ev[k][2 * b + 1]
        return evs

    timed_ev = [timed_events(k) for k in range(args.steps)]
    torch.cuda.synchronize()
    sampler = ClockSampler(local_rank)
    sampler.start()

    def load_step():
        flush.zero_()
        step(warm_ev)

    keep_busy(load_step, LOAD_WINDOW_S, torch.cuda.synchronize)  # the sampler sees the GPU under load
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    for k in range(args.steps):
        flush.zero_()
        starts[k].record(stream)
        step(timed_ev[k])
        ends[k].record(stream)
    torch.cuda.synchronize()
    keep_busy(load_step, LOAD_WINDOW_S, torch.cuda.synchronize)
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop()
    clocks["window"] = f"timed steps plus {LOAD_WINDOW_S:g} s of untimed steps on each side"
    status = dsa.dsa_workspace_status(ws)
    if status != 0:
        raise RuntimeError(f"device status word {status:#x} after the timed steps")

    step_ms = [starts[k].elapsed_time(ends[k]) for k in range(args.steps)]
    total_ms = sum(step_ms)
    sel = dsa.dsa_workspace_selection_stats(ws)  # the last timed step's selection totals
    main_launch_ms = [main_ev[k][2 * b].elapsed_time(main_ev[k][2 * b + 1])
                      for k in range(args.steps) for b in range(nblocks)]
    # Per-stage breakdown (ms per step, summed over query blocks) from untimed
    # steps with an event at every stage boundary (those boundaries serialise
    # the kernels, so these steps run a little longer than the timed ones).
    n_prof = min(args.steps, 10)
    stage_ev = [new_events(EVENTS_PER_BLOCK * nblocks) for _ in range(n_prof)]
    for k in range(n_prof):
        flush.zero_()
        step(stage_ev[k])
    torch.cuda.synchronize()
    stage_names = ["pilot", "threshold", "indexer_main", "select", "fallback", "mla"]
    stages = {n: 0.0 for n in stage_names}
    for k in range(n_prof):
        for b in range(nblocks):
            ev = stage_ev[k][EVENTS_PER_BLOCK * b: EVENTS_PER_BLOCK * (b + 1)]
            for i, n in enumerate(stage_names):
                stages[n] += ev[i].elapsed_time(ev[i + 1]) / n_prof
    total_ms = max_over_ranks(total_ms, world, dev)
    ms_per_step = total_ms / args.steps
    value = job_throughput(cfg.L, world, args.steps, total_ms)

    # ---- end to end through the public API with host buffers (pinned), copies inside the timed region.
    # Every step copies all of its inputs host -> device and reads its whole output back; the copies of
    # step i + 1 run on their own stream while step i computes and its output is read back (two input and
    # output buffers, three streams), as a serving loop would.
    host = {k: v.pin_memory() for k, v in inp.items()}
    out_host = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = out_host[0].numel() * out_host[0].element_size()
    gbuf = [g, {k: torch.empty_like(v) for k, v in g.items()}]
    outs = [out, torch.empty_like(out)]
    s_h2d, s_d2h = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    e2e_steps = max(2, min(args.steps, 10))

    def e2e_run(nsteps, start_event=None):
        if start_event is not None:
            s_h2d.wait_event(start_event)
            s_d2h.wait_event(start_event)
        h2d_done = [torch.cuda.Event() for _ in range(nsteps)]
        comp_done = [torch.cuda.Event() for _ in range(nsteps)]
        d2h_done = [torch.cuda.Event() for _ in range(nsteps)]
        for i in range(nsteps):
            b = i % 2
            with torch.cuda.stream(s_h2d):
                if i >= 2:
                    s_h2d.wait_event(comp_done[i - 2])  # the step that last read buffer b is done
                for k2, v in host.items():
                    gbuf[b][k2].copy_(v, non_blocking=True)
                h2d_done[i].record(s_h2d)
            stream.wait_event(h2d_done[i])
            if i >= 2:
                stream.wait_event(d2h_done[i - 2])  # output buffer b has been read back
            gb = gbuf[b]
            dsa.dsa_prefill_chunk(gb["q_idx"], gb["k_idx"], gb["w"], gb["q"], gb["kv"], cfg.q_pos0, cfg.topk,
                                  cfg.scale, outs[b], workspace=ws, stream=stream)
            comp_done[i].record(stream)
            with torch.cuda.stream(s_d2h):
                s_d2h.wait_event(comp_done[i])
                out_host[b].copy_(outs[b], non_blocking=True)
                d2h_done[i].record(s_d2h)
        stream.wait_event(d2h_done[nsteps - 1])

    e2e_run(2)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    e2e_run(e2e_steps, start_event=e0)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    e2e_value = job_throughput(cfg.L, world, e2e_steps, e2e_ms)

    # ---- roofline of the dominant kernel (main indexer pass: tensor-core contraction)
    fb = flops_and_bytes(cfg)
    peaks = measured_peaks()
    main_ms = statistics.mean(main_launch_ms)
    launches_per_step = nblocks
    idx_flop_per_launch = fb["indexer_flop"] / launches_per_step
    achieved = idx_flop_per_launch / (main_ms / 1000.0) / 1e12
    fp8_peak = measure_fp8_peak(dev) if cfg.idx_dtype == "e4m3" else None
    if cfg.idx_dtype != "e4m3":
        peak, peak_source = peaks["bf16_tflops"], f"{peaks['source']} bf16 burst"
    elif fp8_peak is not None:
        peak, peak_source = fp8_peak, "measured live: torch._scaled_mm e4m3 8192^3, best of 10"
    else:
        peak, peak_source = 2.0 * peaks["bf16_tflops"], f"{peaks['source']} bf16 burst x2 nominal fp8 ratio"
    traffic = indexer_kernel_traffic(cfg)
    # whole-path roofline: max(tensor time at peak, algorithmic bytes at HBM bandwidth)
    t_tensor = (fb["indexer_flop"] / (peak * 1e12)) + fb["mla_flop"] / (peaks["bf16_tflops"] * 1e12)
    # (the indexer FLOPs at their own dtype's peak, the attention FLOPs at the bf16 peak)
    t_bytes = fb["alg_bytes"] / (peaks["hbm_gbs"] * 1e9)
    path_roof_s = max(t_tensor, t_bytes)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        threads = os.cpu_count() or 1
        n_rows = max(4, min(cfg.L, 16 * threads))  # about 10-15 s of wall time on the 128K workload
        rows = sample_rows(cfg, n_rows)
        rate, secs = cpu_oracle_rate(cfg, inp, rows, threads)
        rows1 = sample_rows(cfg, 8, salt=77)  # a few seconds on one core
        rate1, secs1 = cpu_oracle_rate(cfg, inp, rows1, 1)
        cpu = {"value": rate, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": f"{len(rows)} seeded-random query rows of {cfg.name} (full indexer row, exact top-k, "
                         f"attention), {secs:.1f} s wall on {threads} threads",
               "single_core": {"value": rate1, "unit": UNIT, "cores": 1,
                               "sample": f"{len(rows1)} seeded-random query rows, {secs1:.1f} s on one thread"}}

    pilot_launches = 1 if cfg.q_pos0 + min(cfg.L, 1024) > 8192 else 0
    # Per query block: [pilot], threshold, main pass, select, fallback, attention; a chunk with
    # fewer (query, 64-head group) items than half the SMs runs split-key attention plus a merge.
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    split = 2 * cfg.L * ((cfg.H + 63) // 64) <= sms and cfg.topk > 128
    gpu_launches = args.steps * nblocks * (5 + pilot_launches + (1 if split else 0))
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step,
        "ms_per_step_median": statistics.median(step_ms), "ms_per_step_best": min(step_ms),
        "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": cfg.idx_dtype if cfg.idx_dtype == "bf16" else "fp8-e4m3 indexer / bf16 MLA",
        "data": "synthetic",
        "config": {"workload": cfg.name, "N": cfg.N, "L": cfg.L, "topk": cfg.topk, "H": cfg.H, "H_I": cfg.H_I,
                   "D_I": cfg.D_I, "indexer_dtype": cfg.idx_dtype, "query_block": 1024,
                   "l2": "flushed before every timed step (512 MiB device write, outside the step events)",
                   "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "kernel": "indexer_kernel (main pass)",
                     "peak_source": peak_source,
                     "path_frac": path_roof_s / (ms_per_step / 1000.0)},
        "selection": {"candidates_per_query": sel["candidates"] / max(1, sel["queries"]),
                      "max_candidates": sel["max_candidates"], "fallback_queries": sel["fallback_queries"],
                      "queries": sel["queries"], "of": "the last timed step"},
        "stages_ms": {k: round(v, 4) for k, v in stages.items()},
        "stages_from": f"{n_prof} untimed steps with an event at every stage boundary",
        "clocks": clocks,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps, "copies": "pinned host buffers; step i+1's host-to-device copies overlap "
                                              "step i's compute and read-back (3 streams, 2 buffer sets)"},
        "gpu_launches": gpu_launches,
        "cpu_baseline": cpu,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


def run_crossover(args) -> None:
    """Dense-vs-sparse crossover (measurement only, one JSON line per context length).

    For a 1,024-query chunk at the end of an N-key cache (the 128K workload's
    distributions, k = 2,048, 64 heads): the whole sparse path
    (dsa_prefill_chunk) against dense causal attention over every visible key,
    run through the same tcgen05 attention kernel with all visible keys
    selected.  CUDA events, L2 flushed before every timed call.
    """
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    import deepseek_sparse_attention_relu_b200 as dsa
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def timed(fn, reps=5, warm=3):
        for _ in range(warm):
            fn()
        ts = []
        for _ in range(reps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        return statistics.median(ts)

    for N in (2048, 4096, 8192, 16384, 32768, 65536, 131072):
        L = 1024
        cfg = dsa_inputs.small_variant(dsa_inputs.CTX128K, N=N, L=L, topk=2048, H=64)
        g = {k: v.to(dev) for k, v in dsa_inputs.generate(cfg).items()}
        out = torch.empty(L, cfg.H, 512, dtype=torch.bfloat16, device=dev)
        ws = dsa.alloc_workspace(dsa.dsa_prefill_chunk_workspace(L, N, cfg.H_I, cfg.D_I, cfg.H, cfg.topk, 0,
                                                                 dsa.DSA_BF16, False), dev)
        sparse_ms = timed(lambda: dsa.dsa_prefill_chunk(g["q_idx"], g["k_idx"], g["w"], g["q"], g["kv"],
                                                        cfg.q_pos0, cfg.topk, cfg.scale, out, workspace=ws))
        # every visible key of query t: 0 .. q_pos0 + t, then -1
        ar = torch.arange(N, dtype=torch.int32, device=dev)
        vis = (cfg.q_pos0 + torch.arange(L, device=dev)).unsqueeze(1)
        dense_idx = torch.where(ar.unsqueeze(0) <= vis, ar.unsqueeze(0), torch.full_like(ar.unsqueeze(0), -1))
        dense_idx = dense_idx.to(torch.int32).contiguous()
        wsd = dsa.alloc_workspace(dsa.dsa_sparse_mla_workspace(L, cfg.H, N), dev)
        dense_ms = timed(lambda: dsa.dsa_sparse_mla_prefill(g["q"], g["kv"], dense_idx, cfg.scale, out,
                                                            workspace=wsd))
        print(json.dumps({"crossover": True, "N": N, "L": L, "topk": cfg.topk, "H": cfg.H,
                          "sparse_path_ms": round(sparse_ms, 4), "dense_attention_ms": round(dense_ms, 4),
                          "dense_over_sparse": round(dense_ms / sparse_ms, 3)}), flush=True)
        del g, out, ws, wsd, dense_idx


def run_overlap(args) -> None:
    """Neighbouring-query overlap of the selections (measurement only, one JSON line per input): for each pair of
    consecutive queries t, t + 1, the union ratio |A u B| / (|A| + |B|) of their top-k sets (0.5 = identical sets,
    1.0 = disjoint).  Packing two queries over their union pays only when this ratio is low."""
    import numpy as np
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    import deepseek_sparse_attention_relu_b200 as dsa
    for cfg in (dsa_inputs.CTX64K, dsa_inputs.CTX128K, dsa_inputs.CTX256K, dsa_inputs.CORRELATED):
        inp = dsa_inputs.generate(cfg, with_mla=False)
        g = {k: v.to(dev) for k, v in inp.items()}
        idx = torch.empty(cfg.L, cfg.topk, dtype=torch.int32, device=dev)
        dsa.dsa_indexer_topk(g["q_idx"], g["k_idx"], g["w"], cfg.q_pos0, cfg.topk, idx)
        h = idx.cpu().numpy()
        ratios = np.empty(cfg.L - 1)
        for t in range(cfg.L - 1):
            a, b = h[t][h[t] >= 0], h[t + 1][h[t + 1] >= 0]
            inter = np.intersect1d(a, b, assume_unique=True).size
            ratios[t] = (a.size + b.size - inter) / (a.size + b.size)
        print(json.dumps({"overlap": True, "workload": cfg.name, "pairs": int(ratios.size),
                          "union_ratio_mean": float(ratios.mean()), "union_ratio_min": float(ratios.min()),
                          "union_ratio_p10": float(np.percentile(ratios, 10)),
                          "shared_keys_mean": float(cfg.topk * (2 - 2 * ratios.mean())),
                          "pairs_at_or_below_0.75": int((ratios <= 0.75).sum())}), flush=True)
        del g, idx


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=dsa_inputs.CTX128K.name, choices=sorted(dsa_inputs.BY_NAME))
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle timing leg")
    ap.add_argument("--crossover", action="store_true",
                    help="measure the dense-vs-sparse crossover instead (JSON line per context length)")
    ap.add_argument("--overlap", action="store_true",
                    help="measure neighbouring queries' selection overlap instead (JSON line per input)")
    ap.add_argument("--dry-run", action="store_true",
                    help="launch and cross-rank plumbing only, on CPU ranks (gloo); no GPU work")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(spawn_ranks(args.gpus, sys.argv[1:]))
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        log(f"[bench] note: WORLD_SIZE={world} but --gpus={args.gpus}; using WORLD_SIZE")
    if args.dry_run:
        run_dry(args, rank, world)
    elif args.crossover:
        if rank == 0:
            run_crossover(args)
    elif args.overlap:
        if rank == 0:
            run_overlap(args)
    elif args.impl == "reference":
        run_reference(args, rank, world)
    else:
        run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
