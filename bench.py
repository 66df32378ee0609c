#!/usr/bin/env python3
"""Benchmark of the fused attention library on B200.

One step is one pass of the whole hot path over one batch of synthetic input
of the headline workload, B=1, H=16, N=16384, d=128 (bf16 inputs): forward and
backward without a mask, then forward and backward with the causal mask.
That is four C-ABI calls and eight kernel launches. The metric is
attention TFLOPS/s, counted as 4*B*H*N^2*d for the forward and 2.5x that for
the backward, each halved under the causal mask.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

Prints one JSON line (rank 0). With N > 1 (launched by torch.distributed.run)
every rank runs an independent replica of the workload: the path needs no
exchange between GPUs, so there is no data-path collective; the only
collectives are the barrier and the max-over-ranks of the timed region.

--impl reference times the fp64 CPU oracle (the slow, plainly correct
definition of the same computation) on the host cores, on a bounded sample of
the same workload each step.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "attention fwd/bwd TFLOPS/s on 1 B200 at N=16k d=128; % of bf16 tensor peak"
UNIT = "TFLOPS/s"
B, H, N, D = 1, 16, 16384, 128
SEED = 3
WORKLOAD = "attention fwd+bwd, B=1 H=16 N=16384 d=128 bf16, non-causal then causal"

# DRAM traffic of one non-causal main backward launch of the workload above
# (B=1, H=16, N=16384, d=128): dram__bytes_read.sum + dram__bytes_write.sum
# from one ncu capture of that very launch shape. None until a capture of the
# current kernel source exists; a number taken on other source is not used.
BWD_TRAFFIC = {"bytes": 404991232 + 221012480, "read": 404991232, "write": 221012480,
               "shape": "B=1 H=16 N=16384 d=128, non-causal, one launch",
               "source_sha256": "fd440b97907b4bc4be779692f9af95a5949f0293d0bf0a21c8b003dffa0f86a8"}
# Dense bf16 tensor-core peak of a B200 as the vendor states it, reported next
# to the fraction of the measured peak.
SPEC_BF16_TFLOPS = 2250.0


def _flops(causal: bool):
    f = 4.0 * B * H * N * N * D
    f = f / 2 if causal else f
    return f, 2.5 * f


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            m = json.load(fh)
        return float(m["bf16_tflops"]), float(m.get("bf16_tflops_sustained", m["bf16_tflops"])), \
            float(m["hbm_gbs"]), "measured"
    except Exception:
        return 1590.0, 1400.0, 6650.0, "fallback"


def _bwd_source_sha():
    h = hashlib.sha256()
    for f in ("fa_bwd.cuh", "fa_ptx.cuh"):
        with open(os.path.join(ROOT, "exact_attention_118_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi clock/throttle samples of one GPU during the timed region.

    Sampling starts before the region: wait_ready() returns once nvidia-smi
    has printed its first sample (it can take most of a second to start).
    Every sample carries its time stamp; stop() keeps the samples taken
    between the wall-clock times the region started and ended."""

    QUERY = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, gpu_index: str):
        self.proc = None
        self.lines = []
        self.reader = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits", "-lms", "20",
                 "-i", gpu_index], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        import threading

        self.reader = threading.Thread(target=self._read, daemon=True)
        self.reader.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line)

    def wait_ready(self, timeout: float = 5.0) -> bool:
        """Wait (at most `timeout` seconds) for the first sample."""
        t = time.time()
        while self.proc is not None and not self.lines and time.time() - t < timeout:
            time.sleep(0.02)
        return bool(self.lines)

    def stop(self, t0: float, t1: float):
        """Summary of the samples stamped within [t0, t1] (wall-clock seconds);
        all samples, marked as such, if none fall there."""
        if self.proc is None:
            return None
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.reader is not None:
            self.reader.join(timeout=5)
        rows = []
        for line in "".join(self.lines).strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((ts, float(f[2]), float(f[3]), f[6:10]))
            except ValueError:
                continue
        inside = [r for r in rows if t0 <= r[0] <= t1]
        window = "timed region"
        if not inside:
            inside, window = rows, "whole sampling period (none inside the timed region)"
        if not inside:
            return None
        reasons = set()
        for r in inside:
            for name, val in zip(self.NAMES, r[3]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r[1] for r in inside), "sm_max_mhz": max(r[2] for r in inside),
                "reasons": sorted(reasons), "samples": len(inside), "window": window}


# ------------------------------------------------------------ rank helpers

def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank float over the default process group (identity when
    there is none or it has one rank). Used for the timed region."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(step_flops: float, world: int, ms_total_max: float, steps: int):
    """(ms per step, whole-job TFLOP/s): every rank runs its own replica, so
    the job's FLOPs are world * step_flops per step, over the slowest rank."""
    ms_per_step = ms_total_max / steps
    return ms_per_step, step_flops * world / (ms_per_step / 1e3) / 1e12


# ------------------------------------------------------------ oracle sample

def _visible_pairs(rows, causal):
    rows = list(rows)
    return sum(r + 1 for r in rows) if causal else len(rows) * N


def oracle_sample(x, head, rows):
    """Time the fp64 oracle on query rows `rows` of one head, forward and
    backward, non-causal and causal. Returns (seconds, algorithmic FLOPs)."""
    from oracle import attention_backward_rows, attention_forward_rows

    flops = 0.0
    t0 = time.perf_counter()
    for causal in (False, True):
        attention_forward_rows(x["q"], x["k"], x["v"], D ** -0.5, causal, [head], rows)
        attention_backward_rows(x["q"], x["k"], x["v"], x["do"], D ** -0.5, causal, [head], rows)
        flops += 4.0 * D * _visible_pairs(rows, causal) * 3.5  # forward + 2.5x backward
    return time.perf_counter() - t0, flops


def _cpu_threads():
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count()


# ------------------------------------------------------------------ arms

def run_reference(args):
    """fp64 CPU oracle, one bounded sample of the workload per step."""
    from workloads import make_inputs

    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    x = make_inputs(B, H, N, D, SEED)  # the workload's own inputs; the sample uses head (0, 0)
    rows_per_step = 512
    for _ in range(args.warmup):
        oracle_sample(x, (0, 0), range(0, rows_per_step))
    total_t, total_f = 0.0, 0.0
    for s in range(args.steps):
        r0 = (s * rows_per_step) % N
        dt, f = oracle_sample(x, (0, 0), range(r0, r0 + rows_per_step))
        total_t += dt
        total_f += f
    value = total_f / total_t / 1e12
    cores = _cpu_threads()
    sample = (f"query rows of head (0,0), {rows_per_step} rows per step "
              f"(rows {0}..{(args.steps * rows_per_step) % N or N}), forward+backward, non-causal and causal")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total_t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "global_batch": B, "seq_len": N, "parallelism": "none (host cores)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_native(args):
    import torch
    import torch.distributed as dist

    import exact_attention_118_b200 as fa
    from workloads import make_inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    # CPU baseline first (rank 0, one GPU only), before the GPU is busy.
    cpu_baseline = None
    x_cpu = make_inputs(B, H, N, D, SEED)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rows = range(0, 4096)
        dt, f = oracle_sample(x_cpu, (0, 0), rows)
        cpu_baseline = {"value": f / dt / 1e12, "unit": UNIT, "cores": _cpu_threads(), "kind": "oracle",
                        "sample": "query rows 0..4095 of head (0,0), forward+backward, non-causal and causal "
                                  f"({dt:.1f} s)"}

    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream
    # Pinned host copies of the step's inputs (for the end-to-end number) and
    # their device-resident counterparts.
    host_in = {k: v.pin_memory() for k, v in x_cpu.items()}
    dev_in = {k: v.to(dev) for k, v in host_in.items()}
    shape = (B, H, N, D)

    def outputs():
        return {
            "o": torch.empty(shape, dtype=torch.bfloat16, device=dev),
            "lse": torch.empty((B, H, N), dtype=torch.float32, device=dev),
            "dq": torch.empty(shape, dtype=torch.bfloat16, device=dev),
            "dk": torch.empty(shape, dtype=torch.bfloat16, device=dev),
            "dv": torch.empty(shape, dtype=torch.bfloat16, device=dev),
        }

    outs = {False: outputs(), True: outputs()}
    ws_bytes = fa.fa_bwd_workspace_size(B, H, N, D)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    scale = D ** -0.5
    q, k, v, do = (dev_in[n].data_ptr() for n in ("q", "k", "v", "do"))

    def check(st, what):
        if st != fa.FA_OK:
            raise RuntimeError(f"{what}: {fa.fa_strerror(st)}")

    def run_pass(causal, ev=None, inp=None, out=None):
        o = outs[causal] if out is None else out
        qp, kp, vp, dop = (q, k, v, do) if inp is None else (inp[n].data_ptr() for n in ("q", "k", "v", "do"))
        if ev is not None:
            ev[4].record(stream)
        check(fa.fa_fwd(qp, kp, vp, o["o"].data_ptr(), o["lse"].data_ptr(), B, H, N, D, scale, int(causal),
                        fa.FA_BF16, sp), "fa_fwd")
        if ev is not None:
            ev[0].record(stream)
            fa.fa_set_bwd_main_events(ev[1].cuda_event, ev[2].cuda_event)
        check(fa.fa_bwd(qp, kp, vp, o["o"].data_ptr(), o["lse"].data_ptr(), dop, o["dq"].data_ptr(),
                        o["dk"].data_ptr(), o["dv"].data_ptr(), ws.data_ptr(), ws_bytes, B, H, N, D, scale,
                        int(causal), sp), "fa_bwd")
        if ev is not None:
            fa.fa_set_bwd_main_events(None, None)
            ev[3].record(stream)

    def step(evs=None):
        run_pass(False, None if evs is None else evs[0])
        run_pass(True, None if evs is None else evs[1])

    fwd_nc, bwd_nc = _flops(False)
    fwd_c, bwd_c = _flops(True)
    step_flops = fwd_nc + bwd_nc + fwd_c + bwd_c

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    check(fa.fa_get_device_error(sp), "warm-up")

    # ---------------------------------------------- device-resident timed region
    def mk():
        e = torch.cuda.Event(enable_timing=True)
        e.record(stream)  # creates the underlying cudaEvent_t
        return e

    evs = [[[mk() for _ in range(5)] for _ in range(2)] for _ in range(args.steps)]
    gpu_id = os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")[local] if os.environ.get(
        "CUDA_VISIBLE_DEVICES") else str(local)
    torch.cuda.synchronize(dev)
    barrier()
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(gpu_id)
    sampler.wait_ready()
    time.sleep(0.1)
    start, stop = mk(), mk()
    t_wall0 = time.time()
    start.record(stream)
    for s in range(args.steps):
        step(evs[s])
    stop.record(stream)
    torch.cuda.synchronize(dev)
    t_wall1 = time.time()
    barrier()
    torch.cuda.synchronize(dev)
    clocks = sampler.stop(t_wall0, t_wall1)
    check(fa.fa_get_device_error(sp), "timed region")
    ms_total = max_over_ranks(start.elapsed_time(stop), dev)
    ms_per_step, value = aggregate(step_flops, world, ms_total, args.steps)

    # per-pass breakdown (events around each call) and the main backward kernel
    def med(xs):
        return statistics.median(xs)

    per = {}
    bwd_main_ms = {False: [], True: []}
    for c in (False, True):
        e = [evs[s][int(c)] for s in range(args.steps)]
        bwd_total = [x[0].elapsed_time(x[3]) for x in e]
        main = [x[1].elapsed_time(x[2]) for x in e]
        bwd_main_ms[c] = main
        per[c] = {"bwd_ms": med(bwd_total), "bwd_main_ms": med(main),
                  "fwd_ms": med([x[4].elapsed_time(x[0]) for x in e])}

    # The forward alone, in a loop of its own that starts after the GPU has
    # idled briefly (a kernel timed alone, as the burst peak was measured);
    # the in-step figures above come from the hot step loop.
    fwd_idle_s = 0.5
    fwd_ms = {}
    for c in (False, True):
        o = outs[c]
        torch.cuda.synchronize(dev)
        time.sleep(fwd_idle_s)
        a, b_ = mk(), mk()
        a.record(stream)
        for _ in range(args.steps):
            check(fa.fa_fwd(q, k, v, o["o"].data_ptr(), o["lse"].data_ptr(), B, H, N, D, scale, int(c),
                            fa.FA_BF16, sp), "fa_fwd")
        b_.record(stream)
        torch.cuda.synchronize(dev)
        fwd_ms[c] = a.elapsed_time(b_) / args.steps

    peak, peak_sus, hbm, peak_kind = _peaks()
    passes = {}
    for c, tag in ((False, "noncausal"), (True, "causal")):
        ff, fb = _flops(c)
        passes[f"fwd_{tag}"] = {"ms": fwd_ms[c], "tflops": ff / fwd_ms[c] / 1e9,
                                "frac_of_peak": ff / fwd_ms[c] / 1e9 / peak,
                                "frac_of_spec": ff / fwd_ms[c] / 1e9 / SPEC_BF16_TFLOPS,
                                "timed": f"alone, {args.steps} launches after {fwd_idle_s} s idle",
                                "in_step_ms": per[c]["fwd_ms"],
                                "in_step_tflops": ff / per[c]["fwd_ms"] / 1e9,
                                "in_step_frac_of_peak": ff / per[c]["fwd_ms"] / 1e9 / peak}
        passes[f"bwd_{tag}"] = {"ms": per[c]["bwd_ms"], "tflops": fb / per[c]["bwd_ms"] / 1e9,
                                "frac_of_peak": fb / per[c]["bwd_ms"] / 1e9 / peak,
                                "frac_of_spec": fb / per[c]["bwd_ms"] / 1e9 / SPEC_BF16_TFLOPS,
                                "timed": "inside the timed step",
                                "main_kernel_ms": per[c]["bwd_main_ms"]}

    # Roofline of the dominant kernel: the main backward kernel, non-causal
    # launch (the largest share of the step), from its own CUDA events.
    main_ms = statistics.mean(bwd_main_ms[False])
    achieved = bwd_nc / (main_ms / 1e3) / 1e12
    traffic = None
    if BWD_TRAFFIC["bytes"] is not None and BWD_TRAFFIC["source_sha256"] == _bwd_source_sha():
        traffic = BWD_TRAFFIC["bytes"]
    # Algorithmic bytes of one launch: Q, K, V, dO read and dK, dV written in
    # bf16, lse2 and D read, and the fp32 dQ accumulator written once.
    alg_bytes = B * H * N * (6 * D * 2 + 2 * 4 + D * 4)
    roofline = {"kernel": "fa_bwd_kernel<128, non-causal> (main backward)", "bound": "tensor",
                "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "traffic": traffic,
                "traffic_shape": BWD_TRAFFIC["shape"] if traffic else None,
                "traffic_over_algorithmic_bytes": traffic / alg_bytes if traffic else None,
                "algorithmic_flops_per_launch": bwd_nc, "algorithmic_bytes_per_launch": alg_bytes,
                "avg_launch_ms": main_ms,
                "peak_kind": f"{peak_kind} bf16 dense (burst); sustained {peak_sus}",
                "frac_of_sustained": achieved / peak_sus,
                "frac_of_spec": achieved / SPEC_BF16_TFLOPS}

    # ---------------------------------------------------- end-to-end (host buffers)
    # A pipelined application loop: each step uploads its inputs from pinned
    # host memory and reads every output back, with uploads on one copy
    # stream and read-backs on another (PCIe is full duplex), both overlapping
    # the kernels of neighbouring steps. Device inputs and outputs are double
    # buffered so step i+1's upload and step i's read-back never touch what a
    # running kernel uses. Every step's copies lie inside the timed region: the
    # first upload waits for the start event and the stop event waits for the
    # last read-back.
    host_out = {c: {n: torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for n, t in outs[c].items()}
                for c in (False, True)}
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = sum(t.numel() * t.element_size() for c in (False, True) for t in host_out[c].values())
    e2e_in = [dev_in, {n: torch.empty_like(t) for n, t in dev_in.items()}]
    e2e_out = [outs, {c: outputs() for c in (False, True)}]
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def e2e_run(n_steps, begin):
        # begin: event on the compute stream that every copy must follow.
        free_in = [begin, begin]       # buffer's last reader done
        read_out = [{False: begin, True: begin}, {False: begin, True: begin}]  # buffer's read-back done
        uploaded = []
        for i in range(min(2, n_steps)):
            up.wait_event(free_in[i])
            with torch.cuda.stream(up):
                for n in ("q", "k", "v", "do"):
                    e2e_in[i][n].copy_(host_in[n], non_blocking=True)
            ev = mk()
            ev.record(up)
            uploaded.append(ev)
        last = []
        for i in range(n_steps):
            bi = i % 2
            stream.wait_event(uploaded[i])
            done = {}
            for c in (False, True):
                stream.wait_event(read_out[bi][c])
                run_pass(c, inp=e2e_in[bi], out=e2e_out[bi][c])
                done[c] = mk()
                done[c].record(stream)
                down.wait_event(done[c])
                with torch.cuda.stream(down):
                    for n, t in e2e_out[bi][c].items():
                        host_out[c][n].copy_(t, non_blocking=True)
                read_out[bi][c] = mk()
                read_out[bi][c].record(down)
            last = [read_out[bi][False], read_out[bi][True]]
            if i + 2 < n_steps:
                up.wait_event(done[True])  # this buffer's inputs are no longer read
                with torch.cuda.stream(up):
                    for n in ("q", "k", "v", "do"):
                        e2e_in[bi][n].copy_(host_in[n], non_blocking=True)
                ev = mk()
                ev.record(up)
                uploaded.append(ev)
        for ev in last:
            stream.wait_event(ev)

    w = mk()
    w.record(stream)
    e2e_run(2, w)
    torch.cuda.synchronize(dev)
    barrier()
    a, b_ = mk(), mk()
    a.record(stream)
    e2e_steps = max(2, args.steps)
    e2e_run(e2e_steps, a)
    b_.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = max_over_ranks(a.elapsed_time(b_), dev) / e2e_steps
    check(fa.fa_get_device_error(sp), "e2e")

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "global_batch": B * world, "seq_len": N, "heads": H, "head_dim": D,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": "inputs larger than L2 (Q,K,V,dO 67 MB each; 1.1 GB working set per step)"},
        "frac_of_peak": value / peak,
        "frac_of_spec": value / SPEC_BF16_TFLOPS,
        "peak": {"bf16_tflops": peak, "kind": peak_kind, "spec_bf16_tflops": SPEC_BF16_TFLOPS},
        "passes": passes,
        "roofline": roofline,
        "cpu_baseline": cpu_baseline,
        "e2e": {"value": step_flops * world / (e2e_ms / 1e3) / 1e12, "unit": UNIT, "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": 8 * args.steps,
        "clocks": clocks,
        "context": "pages' figure: FlashAttention-2 ~338 TFLOPS/s non-causal at 16k on H100 SXM5 (other hardware)",
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_profile_case(args):
    """Untimed forward+backward launches for an ncu capture: B=1, N=16384,
    d=128, `--profile-case` heads, non-causal (or causal with --causal), three
    passes. Prints nothing but "ok"."""
    import torch

    import exact_attention_118_b200 as fa

    h = args.profile_case
    g = torch.Generator(device="cuda")
    g.manual_seed(0)
    q, k, v, do = (torch.randn(B, h, N, D, device="cuda", generator=g).to(torch.bfloat16) for _ in range(4))
    ws = torch.empty(fa.fa_bwd_workspace_size(B, h, N, D), dtype=torch.uint8, device="cuda")
    for _ in range(3):
        o, lse = fa.attention_forward(q, k, v, causal=args.causal)
        fa.attention_backward(q, k, v, o, lse, do, causal=args.causal, workspace=ws)
    torch.cuda.synchronize()
    fa.check_device_error()
    print("ok")
    return 0


def run_next_rows(args):
    """The widened rows on one GPU, one JSON line each (not part of the default
    run): grouped K/V heads (H_kv = 4 and 1), a 4096-key sliding window, a
    packed variable-length batch and the FP8 forward, all at d = 128 with 16
    query heads and inputs larger than L2. Device-timed with CUDA events over
    --steps calls after --warmup; TFLOP/s count only the visible (query, key)
    pairs: 4 d per pair forward, 2.5 times that backward."""
    import numpy as np
    import torch

    import exact_attention_118_b200 as fa

    peak, _, _, peak_kind = _peaks()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    sp = torch.cuda.current_stream(dev).cuda_stream
    g = torch.Generator(device="cuda")
    g.manual_seed(11)
    d, H = 128, 16
    scale = d ** -0.5

    def rnd(*shape):
        return torch.randn(*shape, device=dev, generator=g).to(torch.bfloat16)

    # Each row starts after the GPU has idled briefly, so that a row's
    # figure does not depend on how hot the rows before it left the part
    # (under the 1 kW power cap the SM clock drops during long busy spells).
    cooldown_s = 0.25

    def timed(fn):
        torch.cuda.synchronize()
        time.sleep(cooldown_s)
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(args.steps):
            fn()
        b.record()
        torch.cuda.synchronize()
        fa.check_device_error()
        return a.elapsed_time(b) / args.steps

    def check(st):
        if st != fa.FA_OK:
            raise RuntimeError(fa.fa_strerror(st))

    def pairs(L, wl, wr):
        i = np.arange(L)
        lo = np.zeros(L) if wl < 0 else np.maximum(0, i - wl)
        hi = np.full(L, L - 1) if wr < 0 else np.minimum(L - 1, i + wr)
        return float(np.sum(hi - lo + 1))

    def emit(row, config, ms_f, ms_b, vis_pairs, dtype="bf16", fwd_peak=None):
        ff = 4.0 * d * H * vis_pairs
        line = {"row": row, "metric": "attention TFLOPS/s of visible work", "unit": UNIT, "dtype": dtype,
                "data": "synthetic", "config": config, "steps": args.steps, "warmup": args.warmup,
                "idle_before_each_pass_s": cooldown_s, "fwd_ms": ms_f, "fwd_tflops": ff / ms_f / 1e9}
        line["fwd_frac_of_peak"] = line["fwd_tflops"] / (fwd_peak or peak)
        if ms_b is not None:
            line.update({"bwd_ms": ms_b, "bwd_tflops": 2.5 * ff / ms_b / 1e9,
                         "bwd_frac_of_peak": 2.5 * ff / ms_b / 1e9 / peak,
                         "value": 3.5 * ff / (ms_f + ms_b) / 1e9})
        else:
            line["value"] = line["fwd_tflops"]
        line["peak"] = fwd_peak or peak
        line["peak_kind"] = peak_kind if fwd_peak is None else f"{peak_kind} bf16 x 2 (nominal e4m3:bf16 ratio)"
        print(json.dumps(line), flush=True)

    # Host cost of one call on the two small workloads (forward of B=1 H=2
    # N=256 d=64 with fp32 O; forward + backward of causal B=2 H=8 N=1024
    # d=64): wall-clock microseconds per call for the host side alone
    # (argument checks, tensor-map encoding, launches; the calls are enqueued
    # behind a sleeping kernel), and with a stream synchronisation after every
    # call (host plus device plus the synchronisation).
    def host_latency(B_, H_, N_, d_, causal, of32):
        x = {n: rnd(B_, H_, N_, d_) for n in ("q", "k", "v", "do")}
        o = torch.empty(B_, H_, N_, d_, device=dev, dtype=torch.float32 if of32 else torch.bfloat16)
        lse = torch.empty(B_, H_, N_, device=dev)
        o16 = torch.empty(B_, H_, N_, d_, device=dev, dtype=torch.bfloat16)
        g3 = [torch.empty_like(x["q"]) for _ in range(3)]
        wsb = fa.fa_bwd_workspace_size(B_, H_, N_, d_)
        ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
        sc = d_ ** -0.5

        def f():
            check(fa.fa_fwd(x["q"].data_ptr(), x["k"].data_ptr(), x["v"].data_ptr(), o.data_ptr(), lse.data_ptr(),
                            B_, H_, N_, d_, sc, causal, fa.FA_F32 if of32 else fa.FA_BF16, sp))

        def b():
            check(fa.fa_bwd(x["q"].data_ptr(), x["k"].data_ptr(), x["v"].data_ptr(), o16.data_ptr(),
                            lse.data_ptr(), x["do"].data_ptr(), g3[0].data_ptr(), g3[1].data_ptr(),
                            g3[2].data_ptr(), ws.data_ptr(), wsb, B_, H_, N_, d_, sc, causal, sp))

        out = {}
        for name, fn in (("fa_fwd", f), ("fa_bwd", b)):
            if of32 and name == "fa_bwd":
                continue
            for _ in range(20):
                fn()
            torch.cuda.synchronize()
            # The host side alone: the stream is held busy by a sleeping
            # kernel, so the calls only enqueue work (n is well below the
            # launch queue's depth) and the time is the library's own.
            n = 100
            torch.cuda._sleep(200_000_000)
            t0 = time.perf_counter()
            for _ in range(n):
                fn()
            t1 = time.perf_counter()
            torch.cuda.synchronize()
            t2 = time.perf_counter()
            m = 200
            for _ in range(m):
                fn()
                torch.cuda.synchronize()
            t3 = time.perf_counter()
            out[name] = {"host_us_per_call": 1e6 * (t1 - t0) / n, "synced_us_per_call": 1e6 * (t3 - t2) / m}
        fa.check_device_error()
        return out

    for tag, args_ in (("fwd_b1h2_n256_d64", (1, 2, 256, 64, 0, True)),
                       ("causal_b2h8_n1024_d64", (2, 8, 1024, 64, 1, False))):
        print(json.dumps({"row": "host_call_latency", "workload": tag, "unit": "us",
                          "calls": host_latency(*args_)}), flush=True)

    N = 16384
    # Grouped K/V heads, causal.
    for Hkv in (4, 1):
        q, do = rnd(1, H, N, d), rnd(1, H, N, d)
        k, v = rnd(1, Hkv, N, d), rnd(1, Hkv, N, d)
        o = torch.empty_like(q)
        lse = torch.empty(1, H, N, device=dev)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        wsb = fa.fa_bwd_gqa_workspace_size(1, H, Hkv, N, d)
        ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
        fwd = lambda: check(fa.fa_fwd_gqa(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),  # noqa: E731
                                          lse.data_ptr(), 1, H, Hkv, N, d, scale, 1, fa.FA_BF16, sp))
        bwd = lambda: check(fa.fa_bwd_gqa(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),  # noqa: E731
                                          lse.data_ptr(), do.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                                          dv.data_ptr(), ws.data_ptr(), wsb, 1, H, Hkv, N, d, scale, 1, sp))
        fwd()
        emit(f"gqa_hkv{Hkv}", {"workload": f"causal grouped-query attention, B=1 H={H} H_kv={Hkv} N={N} d={d}"},
             timed(fwd), timed(bwd), pairs(N, -1, 0))
    # Sliding window.
    wl = 4095
    q, k, v, do = rnd(1, H, N, d), rnd(1, H, N, d), rnd(1, H, N, d), rnd(1, H, N, d)
    o = torch.empty_like(q)
    lse = torch.empty(1, H, N, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    wsb = fa.fa_bwd_gqa_workspace_size(1, H, H, N, d)
    ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
    fwd = lambda: check(fa.fa_fwd_window(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),  # noqa: E731
                                         lse.data_ptr(), 1, H, H, N, d, scale, wl, 0, fa.FA_BF16, sp))
    bwd = lambda: check(fa.fa_bwd_window(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),  # noqa: E731
                                         lse.data_ptr(), do.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                         ws.data_ptr(), wsb, 1, H, H, N, d, scale, wl, 0, sp))
    fwd()
    emit("window_4095_0", {"workload": f"sliding-window causal attention (4096 keys), B=1 H={H} N={N} d={d}"},
         timed(fwd), timed(bwd), pairs(N, wl, 0))
    # Packed variable length: 16 sequences of 512..8192 tokens (seeded), causal.
    lens = [int(x) for x in np.random.default_rng(5).integers(512, 8193, 16)]
    T = sum(lens)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]).astype(np.int32), device=dev)
    q, k, v, do = rnd(T, H, d), rnd(T, H, d), rnd(T, H, d), rnd(T, H, d)
    o = torch.empty_like(q)
    lse = torch.empty(H, T, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    wsb = fa.fa_bwd_varlen_workspace_size(len(lens), T, H, H, d)
    ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
    mx = max(lens)
    fwd = lambda: check(fa.fa_fwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),  # noqa: E731
                                         lse.data_ptr(), cu.data_ptr(), len(lens), mx, T, H, H, d, scale, -1, 0,
                                         fa.FA_BF16, sp))
    bwd = lambda: check(fa.fa_bwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),  # noqa: E731
                                         lse.data_ptr(), do.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                         cu.data_ptr(), ws.data_ptr(), wsb, len(lens), mx, T, H, H, d, scale, -1, 0,
                                         sp))
    fwd()
    emit("varlen_16seq", {"workload": f"packed variable-length causal batch, 16 sequences of 512..8192 tokens "
                                      f"(T={T}, longest {mx}), H={H} d={d}", "lengths": lens},
         timed(fwd), timed(bwd), sum(pairs(L, -1, 0) for L in lens))
    # FP8 forward.
    for causal in (0, 1):
        q8, k8, v8 = ((torch.randn(1, H, N, d, device=dev, generator=g) * 100).to(torch.float8_e4m3fn)
                      .view(torch.uint8) for _ in range(3))
        o = torch.empty(1, H, N, d, dtype=torch.bfloat16, device=dev)
        lse = torch.empty(1, H, N, device=dev)
        fwd = lambda: check(fa.fa_fwd_fp8(q8.data_ptr(), k8.data_ptr(), v8.data_ptr(), o.data_ptr(),  # noqa: E731
                                          lse.data_ptr(), 1, H, H, N, d, scale, 0.01, 0.01, 0.01, -1,
                                          0 if causal else -1, fa.FA_BF16, sp))
        fwd()
        emit(f"fp8_fwd{'_causal' if causal else ''}",
             {"workload": f"FP8 (e4m3) forward{', causal' if causal else ''}, B=1 H={H} N={N} d={d}"},
             timed(fwd), None, pairs(N, -1, 0 if causal else -1), dtype="e4m3", fwd_peak=2.0 * peak)
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-case", type=int, default=0, metavar="HEADS",
                    help="run untimed fwd+bwd launches with this many heads (for ncu) and exit")
    ap.add_argument("--causal", action="store_true", help="with --profile-case: causal mask")
    ap.add_argument("--next-rows", action="store_true",
                    help="time the widened rows (grouped K/V, window, variable length, FP8), one line each")
    args = ap.parse_args()
    if args.next_rows:
        return run_next_rows(args)
    if args.profile_case:
        return run_profile_case(args)
    if args.warmup < 3 and args.impl == "native":
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_native(args)


if __name__ == "__main__":
    sys.exit(main())
