#!/usr/bin/env python3
"""Benchmark: batch-1 greedy decode of the ~1.9B dense decoder (fp16) on one B200 per rank.

Workload (one "step"): the session holds a 1024-token prompt (prefilled once, before
timing); a step rewinds it to those 1024 positions and decodes 512 greedy tokens in one
launch of the persistent megakernel, the argmax fed back on the GPU. Every step streams
all weights (3.65 GB per token) plus the KV cache, far more than the 126 MB L2, so no
L2 flush is needed between steps.

  value     tokens/s over all ranks, device-timed (CUDA events around each launch on the
            launch stream, max over ranks)
  e2e       the same through kie_generate with HOST buffers (doorbell: input token and
            command in, 512 output tokens out), host clock
  roofline  algorithmic bytes per launch / mean launch time, against the measured HBM peak
  cpu_baseline  the CPU oracle's decode steps at this context length on the host cores

Multi-GPU: launched under torchrun, each rank runs an independent replica on its own GPU
(sessions do not shard a single decode; there is no data-path collective).
``--impl reference`` times the CPU oracle instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "batch-1 decode tokens/s and HBM GB/s vs roofline; p99 tick latency at 56 sessions"
PROMPT, DECODE = 1024, 512
WORKLOAD = "dense-1.9b fp16 batch-1 decode: prompt 1024 uniform tokens, greedy decode 512 (28L d2048 16/8x128 F8192 V32000)"


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def algorithmic_bytes(model, ctx0: int, n: int, fp8: bool = False) -> int:
    """Bytes one launch must move: all weights except the embedding table plus one embedding row per token,
    the KV cache read over the attended positions, and the new position's K/V write (fp8: the
    matrices as E4M3 codes plus row scales)."""
    per_pos = model.kv_bytes_per_position()
    total = 0
    for t in range(n):
        attended = ctx0 + t + 1
        total += model.weight_bytes_per_token(fp8) + attended * per_pos + per_pos
    return total


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        import torch
        p = torch.cuda.get_device_properties(device_index)
        self.bus = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.bus, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if not self.proc:
            return None
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        return self.summarise(out)

    @staticmethod
    def summarise(out: str):
        """Median SM clock of the loaded samples (above half the highest), the max clock, and every
        throttle reason seen Active, from `nvidia-smi --format=csv,noheader,nounits` lines of FIELDS."""
        sm, mx, reasons = [], 0.0, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = max(mx, float(parts[1]))
            except ValueError:
                continue
            for name, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):  # "Not Active" does not count
                    reasons.add(name)
        if not sm:
            return None
        loaded = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def oracle_baseline(model, host_weights, ctx0: int, min_s=10.0, max_s=30.0):
    """Decode steps of the CPU oracle at the workload's context length (cache pre-sized, values zero)."""
    from oracle.oracle import OracleModel, num_threads
    orc = OracleModel(model, host_weights, ctx0 + 64)
    orc.pos = ctx0
    tok, steps = 1, 0
    t0 = time.perf_counter()
    while True:
        lg = orc.step(tok)
        tok = int(np.argmax(lg))
        steps += 1
        el = time.perf_counter() - t0
        if el >= min_s or (steps >= 1 and el * (steps + 1) / steps > max_s):
            break
    return {"value": steps / el, "unit": "tokens/s", "cores": num_threads(), "kind": "oracle",
            "sample": f"{steps} oracle decode steps of the full {model.name} model at positions {ctx0}..{ctx0 + steps - 1} "
                      f"(KV cache of that length, zero contents: the per-step cost does not depend on the values)"}


def dist_setup():
    """Rank, world size and local device index under torchrun (one process per GPU): NCCL on
    the rank's GPU, or gloo on a host without CUDA (where only the reference arm can run)."""
    if "RANK" not in os.environ:
        return 0, 1, 0
    import datetime

    import torch
    import torch.distributed as dist
    rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
    local = int(os.environ.get("LOCAL_RANK", rank))
    timeout = datetime.timedelta(seconds=300)
    if torch.cuda.is_available():
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timeout, device_id=torch.device("cuda", local))
    else:
        dist.init_process_group("gloo", timeout=timeout)
    return rank, world, local


def max_over_ranks(x: float, world: int, device="cpu") -> float:
    """The largest of every rank's x (each rank passes its own time; all ranks get the max).
    `device` is where the reduction runs: the rank's GPU under NCCL, the CPU under gloo."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, max_seconds: float) -> float:
    """Throughput of the whole job: the units all ranks processed over the slowest rank's time."""
    return world * units_per_rank / max_seconds


def run_reference(args, rank):
    """The CPU oracle on this arm's workload (the same --model / --prompt / --decode as the engine
    arm): each step is a bounded sample, one greedy decode token of the full model at the
    workload's mean context length, timed on the host cores."""
    if rank != 0:
        return
    from bandwidth_bound_stream_b200 import synth
    from oracle.oracle import OracleModel, num_threads
    m = synth.CONFIGS[args.model]
    prompt_len, decode_n = args.prompt, args.decode
    headline = (args.model == "dense-1.9b" and prompt_len == PROMPT and decode_n == DECODE)
    ctx0 = prompt_len + decode_n // 2
    orc = OracleModel(m, synth.model_weights(m), ctx0 + args.warmup + args.steps + 1)
    orc.pos = ctx0
    tok = 1
    for _ in range(args.warmup):
        tok = int(np.argmax(orc.step(tok)))
    t0 = time.perf_counter()
    for _ in range(args.steps):
        tok = int(np.argmax(orc.step(tok)))
    el = time.perf_counter() - t0
    value = args.steps / el
    sample = (f"{args.steps} timed oracle decode steps (after {args.warmup} warm-up) of the full {m.name} model at "
              f"positions {ctx0 + args.warmup}.. (KV cache of that length, zero contents)")
    cb = {"value": value, "unit": "tokens/s", "cores": num_threads(), "kind": "oracle", "sample": sample}
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(el / args.steps * 1e3, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD if headline else f"{m.name} batch-1: prompt {prompt_len}, decode {decode_n}",
                       "prompt": prompt_len, "decode": decode_n, "batch": 1,
                       "parallelism": "CPU oracle, OpenMP over output rows",
                       "step": "one decode token of the workload per step (bounded sample)"},
            "cpu_baseline": cb,
            "e2e": {"value": round(value, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="engine", choices=["engine", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--model", default="dense-1.9b", help="workload shape (profiling cases use smaller ones)")
    ap.add_argument("--prompt", type=int, default=PROMPT)
    ap.add_argument("--decode", type=int, default=DECODE)
    ap.add_argument("--ticks", type=int, default=500, help="timed ticks of the 56-session workload (0 = skip)")
    ap.add_argument("--tick-only", action="store_true", help="only the tick workload (its own JSON line)")
    ap.add_argument("--no-extra", action="store_true", help="skip the 8B and 32K-context batch-1 workloads")
    ap.add_argument("--b1-staging", type=int, default=0, choices=[0, 1],
                    help="batch-1 weight staging: 0 = shared-memory ring, 1 = ring plus TMEM slots for the attention step")
    ap.add_argument("--extra-steps", type=int, default=3, help="timed launches of each extra workload")
    ap.add_argument("--tick-model", default="dense-10.8b")
    ap.add_argument("--tick-prompt", type=int, default=0, help="fixed prompt length per session (0 = seeded 1000-1500)")
    ap.add_argument("--trace", type=int, default=0,
                    help="after the timed region, trace this many tokens (<= 8) of one more launch and add the "
                         "batch-1 kernel's per-phase durations as phase_us (0 = off)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    rank, world, local = dist_setup()
    if args.tick_only:
        import torch
        torch.cuda.set_device(local)
        t = run_tick(args.ticks, args.warmup, local, clocks_for=local, model_name=args.tick_model,
                     prompt_len=args.tick_prompt)
        if rank == 0:
            print(json.dumps({"metric": "p99 tick latency at 56 sessions", "value": t["p99_ms"], "unit": "ms",
                              "higher_is_better": False, "n_gpus": world, "tick": t}), flush=True)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    if args.impl == "reference":
        run_reference(args, rank)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return

    import torch

    from bandwidth_bound_stream_b200 import kie, synth
    m = synth.CONFIGS[args.model]
    prompt_len, decode_n = args.prompt, args.decode
    headline = (args.model == "dense-1.9b" and prompt_len == PROMPT and decode_n == DECODE)
    dev = f"cuda:{local}"
    torch.cuda.set_device(local)
    want_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline
    dw = kie.DeviceWeights(m, seed=0, device=dev, host_copy=want_cpu)
    prompt = synth.prompt(m, prompt_len)
    # both kernels: the prompt is prefilled in chunks of 64 positions on the tensor cores
    eng = kie.Engine(kie.config(m, max_ctx=prompt_len + decode_n, timeout_ms=10000, idle_ms=200, device=local,
                                modes=kie.KIE_MODE_BATCH1 | kie.KIE_MODE_TICK, b1_staging=args.b1_staging), dw.kie)
    host_weights = dw.host
    dw.free()  # the engine keeps its own repacked copy
    torch.cuda.empty_cache()
    sid = eng.session_open()
    t0 = time.perf_counter()
    first = eng.prefill(sid, prompt)
    ttft_ms = (time.perf_counter() - t0) * 1e3

    stream = torch.cuda.Stream(device=dev)
    tok_d = torch.tensor([first], dtype=torch.int32, device=dev)
    out_d = torch.zeros(decode_n, dtype=torch.int32, device=dev)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]

    def launch():
        eng.session_rewind(sid, prompt_len)
        eng.decode_launch(sid, tok_d.data_ptr(), decode_n, out_d.data_ptr(), None, stream.cuda_stream)

    for _ in range(args.warmup):
        launch()
    eng.sync()
    ref_tokens = out_d.cpu().numpy().copy()
    agreements = []
    torch.cuda.nvtx.range_push("kie_decode_timed")

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    clocks = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    t_all0 = torch.cuda.Event(enable_timing=True)
    t_all1 = torch.cuda.Event(enable_timing=True)
    t_all0.record(stream)
    for i in range(args.steps):
        starts[i].record(stream)
        launch()
        ends[i].record(stream)
    t_all1.record(stream)
    torch.cuda.nvtx.range_pop()
    eng.sync()
    torch.cuda.synchronize()
    clock_info = clocks.stop()
    barrier()
    total_ms = t_all0.elapsed_time(t_all1)
    per_launch = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    # the residual's fp32 atomic adds may round in a different order from launch to launch, which
    # can flip an argmax whose top two logits are within ~1e-6 (then the rest of the chain differs)
    agreements.append(float(np.mean(out_d.cpu().numpy() == ref_tokens)))
    total_ms = max_over_ranks(total_ms, world, dev)

    # end to end through the doorbell with host buffers
    out_h = np.empty(decode_n, dtype=np.int32)
    for _ in range(2):
        eng.session_rewind(sid, prompt_len)
        eng.generate(sid, first, decode_n, out_h)
    barrier()
    e0 = time.perf_counter()
    for _ in range(args.steps):
        eng.session_rewind(sid, prompt_len)
        eng.generate(sid, first, decode_n, out_h)
    e_s = time.perf_counter() - e0
    agreements.append(float(np.mean(out_h == ref_tokens)))
    assert out_h.min() >= 0 and out_h.max() < m.vocab
    e_s = max_over_ranks(e_s, world, dev)

    # inter-token latency of single doorbell steps (host clock)
    eng.session_rewind(sid, prompt_len)
    itl = []
    tok = first
    for _ in range(min(64, decode_n)):
        a = time.perf_counter()
        tok = eng.decode_step(sid, tok)
        itl.append((time.perf_counter() - a) * 1e3)
    phase_us = None
    if args.trace > 0:  # untimed: one more launch with the phase trace on, at the same context
        from bandwidth_bound_stream_b200 import trace
        n_tr = min(args.trace, 8, decode_n)
        eng.trace_enable(n_tr)
        eng.session_rewind(sid, prompt_len)
        eng.decode_launch(sid, tok_d.data_ptr(), n_tr, out_d.data_ptr(), None, stream.cuda_stream)
        eng.sync()
        phase_us = trace.batch1_phase_us(eng.trace_read(n_tr), m.n_layers)
        eng.trace_enable(0)
    eng.close()

    value = whole_job_rate(decode_n * args.steps, world, total_ms / 1e3)
    peak, peak_kind = measured_peaks()
    bytes_launch = algorithmic_bytes(m, prompt_len, decode_n)
    mean_launch_s = statistics.mean(per_launch) / 1e3
    achieved = bytes_launch / mean_launch_s / 1e9
    traffic = None
    prof = os.path.join(ROOT, "profiles", "traffic_b1_dense1p9b.json")
    if os.path.exists(prof):
        with open(prof) as f:
            tr = json.load(f)
        if headline and tr.get("kernel_rev") == kernel_revision():
            traffic = tr.get("bytes_per_launch")
    dtype_name = "bf16" if m.dtype == 1 else "fp16"
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": dtype_name, "data": "synthetic",
        "config": {"workload": WORKLOAD if headline else f"{m.name} batch-1: prompt {prompt_len}, decode {decode_n}",
                   "prompt": prompt_len, "decode": decode_n, "batch": 1,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": f"inputs larger than L2 ({m.weight_bytes_per_token() / 1e9:.2f} GB of weights streamed per token);"
                         " no flush needed",
                   "weights": f"seeded N(0,0.02) {dtype_name}, norms 1"},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic, "peak_kind": peak_kind,
                     "bytes_per_launch": bytes_launch, "kernel": f"kie_b1_kernel (one launch = {decode_n} tokens)"},
        "e2e": {"value": round(world * decode_n * args.steps / e_s, 2), "unit": "tokens/s",
                "h2d_bytes_per_step": 4 + 80, "d2h_bytes_per_step": decode_n * 4 + 8,
                "path": "kie_generate via the mapped-mailbox doorbell (host token + command in, host tokens out)"},
        "gpu_launches": args.steps,
        "clocks": clock_info,
        "token_agreement": {"launch_vs_first_launch": agreements[0], "doorbell_vs_launch": agreements[1]},
        "latency": {"ttft_ms": round(ttft_ms, 2), "itl_ms_p50": round(statistics.median(itl), 4),
                    "itl_ms_p99": round(float(np.percentile(itl, 99)), 4),
                    "per_launch_ms": [round(x, 3) for x in per_launch]},
    }
    if phase_us is not None:
        line["phase_us"] = phase_us
    if args.ticks > 0 and headline:
        line["tick"] = run_tick(args.ticks, args.warmup, local, clocks_for=local)
    if headline and not args.no_extra and world == 1:
        line["configs"] = {f"{n}{'-fp8' if f8 else ''}@{p}+{d}": run_extra(n, p, d, f8, args.extra_steps, 3, local, peak,
                                                                             args.b1_staging)
                           for n, p, d, f8 in EXTRA_CONFIGS}
    if want_cpu:
        line["cpu_baseline"] = oracle_baseline(m, host_weights, prompt_len + decode_n // 2)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# The other batch-1 workloads of the method's configurations, measured after the headline in
# the same run (each: its own engine, the prompt prefilled before timing, device-timed launches).
EXTRA_CONFIGS = (("dense-8b", 4096, 256, False), ("dense-1.9b", 32768, 256, False), ("dense-1.9b", 1024, 512, True))


def run_extra(name: str, prompt_len: int, decode_n: int, fp8: bool, steps: int, warmup: int, local: int,
              peak: float, staging: int = 0) -> dict:
    """tokens/s and the roofline of one more batch-1 workload (steps launches of decode_n tokens);
    fp8: the engine streams E4M3 weights with row scales (the prompt then goes through the
    batch-1 kernel as well)."""
    import torch

    from bandwidth_bound_stream_b200 import kie, synth
    m = synth.CONFIGS[name]
    dev = f"cuda:{local}"
    t0 = time.perf_counter()
    dw = kie.DeviceWeights(m, seed=0, device=dev)
    modes = kie.KIE_MODE_BATCH1 if fp8 else kie.KIE_MODE_BATCH1 | kie.KIE_MODE_TICK
    eng = kie.Engine(kie.config(m, max_ctx=prompt_len + decode_n, timeout_ms=20000, idle_ms=200, device=local,
                                modes=modes, weight_fp8=fp8, b1_staging=staging), dw.kie)
    dw.free()
    torch.cuda.empty_cache()
    setup_s = time.perf_counter() - t0
    sid = eng.session_open()
    t0 = time.perf_counter()
    first = eng.prefill(sid, synth.prompt(m, prompt_len))
    ttft_ms = (time.perf_counter() - t0) * 1e3
    stream = torch.cuda.Stream(device=dev)
    tok_d = torch.tensor([first], dtype=torch.int32, device=dev)
    out_d = torch.zeros(decode_n, dtype=torch.int32, device=dev)

    def launch():
        eng.session_rewind(sid, prompt_len)
        eng.decode_launch(sid, tok_d.data_ptr(), decode_n, out_d.data_ptr(), None, stream.cuda_stream)

    for _ in range(warmup):
        launch()
    eng.sync()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    clocks = ClockSampler(local)
    torch.cuda.synchronize()
    clocks.start()
    for a, b in ev:
        a.record(stream)
        launch()
        b.record(stream)
    eng.sync()
    torch.cuda.synchronize()
    clk = clocks.stop()
    per = [a.elapsed_time(b) for a, b in ev]
    eng.close()
    bytes_launch = algorithmic_bytes(m, prompt_len, decode_n, fp8)
    mean_s = statistics.mean(per) / 1e3
    achieved = bytes_launch / mean_s / 1e9
    wt = "E4M3 weights with fp32 row scales, " if fp8 else ""
    return {"workload": f"{name} {wt}{'bf16' if m.dtype else 'fp16'} batch-1: prompt {prompt_len}, greedy decode {decode_n}",
            "tokens_per_s": round(decode_n * steps / (sum(per) / 1e3), 2), "steps": steps, "warmup": warmup,
            "per_launch_ms": [round(x, 3) for x in per],
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "bytes_per_launch": bytes_launch},
            "ttft_ms": round(ttft_ms, 1), "setup_s": round(setup_s, 1), "clocks": clk}


TICK_SESSIONS, TICK_STEPS, TICK_DEADLINE_MS = 56, 2, 160.0


def run_tick(n_ticks: int, warmup: int, local: int, clocks_for: int, model_name: str = "dense-10.8b",
             prompt_len: int = 0) -> dict:
    """The continuous-inference workload: 56 sessions of the 10.8B bf16 model, each prefilled
    with a seeded prompt of 1000-1500 tokens, then n_ticks ticks of 2 greedy steps per session
    through kie_tick (one doorbell per tick). Tick latency is the host-side round trip of one
    kie_tick call (doorbell written -> outputs read), as a server would see it."""
    import torch

    from bandwidth_bound_stream_b200 import kie, synth
    m = synth.CONFIGS[model_name]
    dev = f"cuda:{local}"
    lens = [prompt_len or synth.tick_prompt_length(s) for s in range(TICK_SESSIONS)]
    max_ctx = max(lens) + TICK_STEPS * (2 * n_ticks + 2 * warmup) + 8
    t0 = time.perf_counter()
    dw = kie.DeviceWeights(m, seed=0, device=dev)
    eng = kie.Engine(kie.config(m, max_sessions=TICK_SESSIONS, max_ctx=max_ctx, timeout_ms=60000, idle_ms=500,
                                device=local, modes=kie.KIE_MODE_TICK), dw.kie)
    dw.free()
    torch.cuda.empty_cache()
    setup_s = time.perf_counter() - t0
    sids = [eng.session_open() for _ in range(TICK_SESSIONS)]
    t0 = time.perf_counter()
    tokens = np.array([eng.prefill(sids[s], synth.prompt(m, lens[s], session=s)) for s in range(TICK_SESSIONS)],
                      dtype=np.int32)
    prefill_s = time.perf_counter() - t0
    for _ in range(warmup):
        tokens = eng.tick(sids, tokens, TICK_STEPS)[-1].copy()
    ctx0 = [eng.session_length(s) for s in sids]
    clocks = ClockSampler(clocks_for)
    clocks.start()
    lat = []
    for _ in range(n_ticks):
        a = time.perf_counter()
        out = eng.tick(sids, tokens, TICK_STEPS)
        lat.append((time.perf_counter() - a) * 1e3)
        tokens = out[-1].copy()
    clk = clocks.stop()
    # the same ticks, stream-ordered on device buffers and timed with CUDA events (device time),
    # from the same contexts: the sessions are rewound to where the doorbell ticks started (else
    # every tick would attend ~2 * n_ticks more positions)
    for s, c in zip(sids, ctx0):
        eng.session_rewind(s, c)
    stream = torch.cuda.Stream(device=dev)
    tok_d = torch.tensor(tokens, device=dev)
    outs = [torch.zeros((TICK_STEPS, TICK_SESSIONS), dtype=torch.int32, device=dev) for _ in range(2)]
    for k in range(warmup):
        eng.tick_launch(sids, tok_d.data_ptr() if k == 0 else outs[(k - 1) % 2][-1].data_ptr(), TICK_STEPS,
                        outs[k % 2].data_ptr(), None, stream.cuda_stream)
    eng.sync()
    for s, c in zip(sids, ctx0):
        eng.session_rewind(s, c)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_ticks)]
    torch.cuda.nvtx.range_push("kie_tick_timed")
    for k in range(n_ticks):
        src = outs[(warmup + k - 1) % 2][-1] if warmup + k > 0 else tok_d
        ev[k][0].record(stream)
        eng.tick_launch(sids, src.data_ptr(), TICK_STEPS, outs[(warmup + k) % 2].data_ptr(), None, stream.cuda_stream)
        ev[k][1].record(stream)
    torch.cuda.nvtx.range_pop()
    eng.sync()
    dev_ms = np.array([a.elapsed_time(b) for a, b in ev])
    eng.close()
    lat = np.array(lat)
    # bytes one tick must move: all weights but the embedding table (plus one row per session) per
    # step, each session's KV read over its attended positions, and its new K/V write
    per_pos = m.kv_bytes_per_position()
    tick_bytes = []
    for k in range(n_ticks):
        b = 0
        for st in range(TICK_STEPS):
            b += m.weight_bytes_per_token() + (TICK_SESSIONS - 1) * 2 * m.d_model
            b += sum((c + TICK_STEPS * k + st + 1) * per_pos + per_pos for c in ctx0)
        tick_bytes.append(b)
    gbs = float(np.median(np.array(tick_bytes) / (lat / 1e3)) / 1e9)
    misses = int((lat > TICK_DEADLINE_MS).sum())
    shape = (f"{m.name} {'bf16' if m.dtype == 1 else 'fp16'} ({m.n_layers}L d{m.d_model} "
             f"{m.n_heads}/{m.n_kv_heads}x{m.head_dim} F{m.ffn} V{m.vocab})")
    return {"model": shape, "sessions": TICK_SESSIONS,
            "steps_per_tick": TICK_STEPS, "ticks": n_ticks, "session_ticks": TICK_SESSIONS * n_ticks,
            "ctx_start_range": [min(lens), max(lens)], "p50_ms": round(float(np.percentile(lat, 50)), 3),
            "p99_ms": round(float(np.percentile(lat, 99)), 3), "max_ms": round(float(lat.max()), 3),
            "deadline_ms": TICK_DEADLINE_MS, "ticks_late": misses, "session_ticks_late": misses * TICK_SESSIONS,
            "achieved_gbs_median": round(gbs, 1), "prefill_s": round(prefill_s, 2), "setup_s": round(setup_s, 1),
            "device_ms_p50": round(float(np.percentile(dev_ms, 50)), 3),
            "device_ms_p99": round(float(np.percentile(dev_ms, 99)), 3),
            "device_launches": n_ticks,
            "path": "kie_tick via the mapped-mailbox doorbell, host clock", "clocks": clk}


def kernel_revision() -> str:
    """Hash of the kernel sources (traffic counters are valid only for the revision they were taken on)."""
    import hashlib
    h = hashlib.sha1()
    csrc = os.path.join(ROOT, "bandwidth_bound_stream_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.startswith("kie_b1") or name in ("kie_device.cuh", "kie_attn.cuh", "kie_internal.h",
                                                  "kie_sample.cuh"):
            with open(os.path.join(csrc, name), "rb") as f:
                h.update(f.read())
    return h.hexdigest()[:12]


if __name__ == "__main__":
    main()
