#!/usr/bin/env python
"""Throughput benchmark of the RWKV-7 (x070) state-recurrence library on B200.

A step is one prefill call over one batch of the 7.2B-width long-context workload
(D4096: B=4 sequences x T=16384 tokens x H=64 heads of size 64, bf16 operands with
the slow-decay generator z ~ N(1, 1), float32 state out, zero initial state).  It
is the largest of the single-GPU workloads, so the headline is quoted on it.  The
kernel reads the six operand tensors and writes y and the final state: 3.76 GB per
step, far larger than the 126 MB L2, so no L2 flush is needed between steps.

One JSON line is printed by rank 0:
  value      prefill tokens/s over all ranks (device time, CUDA events, max over ranks)
  e2e        the same metric through the C-ABI call with host buffers
             (rwkv7_wkv_prefill_host_bf16): pinned host -> device copies of the
             operands, the prefill, and device -> host copies of y and the final
             state, in batch slices whose copies overlap the compute of other
             slices; all timed
  roofline   the prefill kernel's algorithmic HBM bytes / its average launch time
  configs    every workload timed the same way, each with its own roofline:
             the float32 B1 T64 H2 case, the 0.1B-shape prefill, the 1.5B-shape
             two-call chain, the L24-D1024 decode (fresh tokens every step, float32
             and bfloat16 state), the 7.2B-width prefill and its ragged batch
  schedules  the opt-in pipelined chunk schedule on two of those workloads
  cpu_baseline  the float64 oracle on this host's cores (rank 0, N=1 only) on a
             bounded sample of the headline workload

Inputs are drawn on the device with the seeded recipe of ``wkv7_inputs`` (same
distributions as the CPU draws the parity tests use, different random stream).

Multi-GPU (torchrun): every rank runs its own batch (weak scaling); the
recurrence has no cross-rank exchange, so the only collectives are the
barrier and the max-reduction of the timings.

``--impl reference`` times the float64 CPU oracle instead (the only other
program this workload has), on rank 0, on a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import wkv7_inputs as wi  # noqa: E402

N = 64
OPS = ("r", "w", "k", "v", "a", "b")
NATIVE = ("r", "xw", "k", "v", "xa")
HEADLINE = "prefill_d4096_b4_t16384"
SMALL = "prefill_d768_b8_t4096"          # the option and training legs run on this shape
RAGGED_LO, RAGGED_HI = 1024, 16384       # per-row lengths of the 7.2B-width ragged batch
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per token-head of one chunk-kernel launch
# with one CTA per (b, h) pair, from one ncu capture of the headline shape at B=1 (64 pairs, 940 MB of
# operands, larger than L2) forced to that schedule, scaled by the token-heads of a launch; the figure
# holds only for the kernel source it was taken on (sha256 prefix of wkv7_chunk.cu), and the line
# reports null for any other build.  The capture is summarised under profiles/.
MEASURED_TRAFFIC = {"source_sha256": "ec571157ca8177a4", "bytes_per_token_head": (805728000 + 124227584) / (16384 * 64)}


def measured_traffic(B, T, H, schedule):
    import hashlib
    if MEASURED_TRAFFIC["source_sha256"] is None or schedule not in ("auto", "pair"):
        return None
    src = os.path.join(ROOT, "rwkv_delta_rule_b200", "csrc", "wkv7_chunk.cu")
    try:
        with open(src, "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()[:16]
    except OSError:
        return None
    if sha != MEASURED_TRAFFIC["source_sha256"]:
        return None
    return MEASURED_TRAFFIC["bytes_per_token_head"] * B * T * H


def prefill_bytes(tokens, H, B, elem=2, state_in=True, n_ops=6):
    """Algorithmic HBM bytes of one prefill call over `tokens` token rows (B*T, or the packed total of
    a ragged batch): `n_ops` operands read and y written (tokens*H*N elements each), the final state
    written and, when there is one, the initial state read (B*H*N*N float32 each)."""
    return (n_ops + 1) * tokens * H * N * elem + (2 if state_in else 1) * B * H * N * N * 4


def decode_bytes(B, H, elem=2, state_elem=4, n_ops=6):
    """Algorithmic HBM bytes of one decode step: state read + written, `n_ops` operand vectors read,
    y written."""
    return B * H * (2 * N * N * state_elem + (n_ops + 1) * N * elem)


# Prefill FLOPs per token-head of the chunked form at a fixed reference chunk C = 64 (so that the choice
# of chunk size cannot move the figure): 2 (8 C N + 4 N^2 + C^2 / 6) = 99.7 kflop
PREFILL_FLOP_PER_TOKEN_HEAD = 2 * (8 * 64 * N + 4 * N * N + 64 * 64 / 6)


def tensor_view(tokens, H, ms, peaks):
    """The same launch against the tensor-core bound: algorithmic FLOPs at C = 64 over the launch time,
    against the measured dense bf16 peak (the products run in bf16 and tf32; tf32 has half that peak,
    so this fraction is an upper bound of the tensor pipe's share)."""
    flops = PREFILL_FLOP_PER_TOKEN_HEAD * tokens * H
    tf = flops / (ms / 1e3) / 1e12
    return {"bound": "tensor", "achieved": tf, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
            "frac": tf / peaks["bf16_tflops"], "flops_per_launch": flops}


def training_bytes(B, T, H):
    """Algorithmic HBM bytes of the training pair over B x T tokens and H heads: the checkpointing
    forward reads 6 bf16 operands and the initial state and writes y, a state every 64 tokens and the
    final state; the backward reads the 6 operands, dy, the saved states and ds_out and writes 6
    float32 gradients and ds_in."""
    th, pairs, nck = B * T * H, B * H, -(-T // 64)
    fwd = th * 7 * N * 2 + pairs * (nck + 2) * N * N * 4
    bwd = th * (7 * N * 2 + 6 * N * 4) + pairs * (nck + 2) * N * N * 4
    return fwd, bwd


def hbm_roofline(byts, ms, peaks, **extra):
    achieved = byts / (ms / 1e3) / 1e9
    out = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
           "frac": achieved / peaks["hbm_gbs"], "algorithmic_bytes_per_launch": byts, "launch_ms": ms}
    out.update(extra)
    return out


class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi during a timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int, path: str | None = None):
        self.device = device
        self.proc = None
        self.path = path

    def __enter__(self):
        sel = []
        try:
            uuid = str(torch.cuda.get_device_properties(self.device).uuid)
            sel = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            sel = []
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", *sel, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]
            if self.path:
                with open(self.path, "w") as f:
                    f.write("\n".join(self.lines) + "\n")
        return False

    def summary(self):
        if not getattr(self, "lines", None):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
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
            for nm, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        # samples taken while the kernels ran: the upper half of the clock samples
        load = sorted(sm)[len(sm) // 2:]
        return {"sm_mhz": statistics.median(load), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def max_over_ranks(x: float, world: int) -> float:
    from rwkv_delta_rule_b200.dist import max_over_ranks as _max

    return x if world == 1 else _max(x)


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def free_device():
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def time_calls(fn, steps, stream, warmup=3):
    """Mean per-call device time (ms) from CUDA events around every call on `stream`, after
    `warmup` untimed calls."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        evs[i][0].record(stream)
        fn()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    return statistics.mean(a.elapsed_time(b) for a, b in evs)


# ---- CPU oracle timing -------------------------------------------------------------------------------

def oracle_sample(T_sample: int, device=None):
    """The bounded oracle sample of the headline workload: batch row 0 (all 64 heads), its first
    `T_sample` tokens, float32 copies of the bf16 operands (exact), zero initial state."""
    case = wi.CASES[HEADLINE]
    d = wi.draw(1, T_sample, case.H, seed=case.seed, dtype=case.dtype, z_mean=case.z_mean, device=device,
                f32_copies=False)
    return [d[n].float().cpu() for n in OPS]


def time_oracle(ops, budget_s: float, min_reps: int = 1):
    """Run the float64 oracle over the sample until about `budget_s` seconds have passed;
    returns (tokens/s, reps, seconds, threads)."""
    import oracle

    B, T = ops[0].shape[0], ops[0].shape[1]
    threads = oracle.default_threads()
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle.wkv7(*ops, None, nthreads=threads)
        reps += 1
        el = time.perf_counter() - t0
        if reps >= min_reps and el >= budget_s:
            break
        if reps >= min_reps and el * (reps + 1) / reps > budget_s * 3:
            break
    return B * T * reps / el, reps, el, threads


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


# ---- reference arm ------------------------------------------------------------------------------------

def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    case = wi.CASES[HEADLINE]
    import oracle

    threads = oracle.default_threads()
    T_sample = min(case.T, args.ref_tokens)
    sub = oracle_sample(T_sample)
    for _ in range(args.warmup):
        oracle.wkv7(*sub, None, nthreads=threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.wkv7(*sub, None, nthreads=threads)
    el = time.perf_counter() - t0
    value = T_sample * args.steps / el
    sample = (f"batch row 0 of {case.B} (all {case.H} heads) x first {T_sample} of {case.T} tokens per step, "
              f"float64 C oracle, {threads} threads ({cpu_model()})")
    line = {
        "impl": "reference", "metric": "wkv7 prefill tokens/s", "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": HEADLINE, "B": case.B, "T": case.T, "H": case.H, "N": N, "global_batch": case.B,
                   "seq_len": case.T, "parallelism": "replicas only", "operands": "bf16 (exact in fp64)"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---- the per-workload legs ----------------------------------------------------------------------------

def bench_f32_small(lib7, dev, steps, peaks):
    """The float32 B1 T64 H2 case (zero initial state): launch-bound, its 0.29 MB stay in L2."""
    case = wi.CASES["prefill_f32_b1_t64_h2"]
    d = wi.draw_case(case)
    dd = {n: d[n].to(dev) for n in OPS}
    y = torch.empty_like(dd["r"])
    s_out = torch.empty(case.B, case.H, N, N, device=dev)
    stream = torch.cuda.current_stream(dev)
    ms = time_calls(lambda: lib7.rwkv7_wkv_prefill(*[dd[n] for n in OPS], None, y, s_out, stream), steps, stream)
    byts = prefill_bytes(case.B * case.T, case.H, case.B, elem=4, state_in=False)
    return {"launch_us": ms * 1e3, "tokens_per_s": case.B * case.T / (ms / 1e3), "dtype": "f32",
            "roofline": hbm_roofline(byts, ms, peaks, l2="0.29 MB per call: L2-resident, launch-bound")}


def bench_prefill(lib7, dev, name, steps, peaks, schedule=0, B=None, T=None):
    """One dense bf16 prefill workload (AUTO path, or a forced chunk schedule)."""
    case = wi.CASES[name]
    B = B or case.B
    T = T or case.T
    d = wi.draw(B, T, case.H, seed=case.seed, dtype="bf16", z_mean=case.z_mean, s0_std=case.s0_std, device=dev,
                f32_copies=False)
    dd = {n: d[n] for n in OPS}
    s0 = d["s0"]
    y = torch.empty_like(dd["r"])
    s_out = torch.empty(B, case.H, N, N, device=dev)
    stream = torch.cuda.current_stream(dev)
    if schedule:
        def fn():
            lib7.rwkv7_wkv_prefill_ext_bf16(lib7.RWKV7_PATH_CHUNK, *[dd[n] for n in OPS], s0, y, s_out,
                                            schedule=schedule, stream=stream)
    else:
        def fn():
            lib7.rwkv7_wkv_prefill_bf16_path(lib7.RWKV7_PATH_AUTO, *[dd[n] for n in OPS], s0, y, s_out, stream)
    ms = time_calls(fn, steps, stream)
    st = lib7.rwkv7_get_last_error()
    byts = prefill_bytes(B * T, case.H, B, state_in=s0 is not None)
    out = {"B": B, "T": T, "H": case.H, "launch_ms": ms, "tokens_per_s": B * T / (ms / 1e3), "status": st,
           "roofline": hbm_roofline(byts, ms, peaks)}
    del d, dd, y, s_out, s0
    free_device()
    return out


def bench_chained(lib7, dev, steps, peaks):
    """The 1.5B-shape chain: two consecutive 4096-token calls, the second starting from the first's
    final state; a step is both calls."""
    case = wi.CASES["prefill_d2048_b16_t8192_chained"]
    B, H, half = case.B, case.H, case.T // 2
    d = wi.draw(B, case.T, H, seed=case.seed, dtype="bf16", z_mean=case.z_mean, device=dev, f32_copies=False)
    parts = [{n: d[n][:, i * half:(i + 1) * half].contiguous() for n in OPS} for i in range(2)]
    del d
    y = [torch.empty_like(parts[0]["r"]) for _ in range(2)]
    s_mid = torch.empty(B, H, N, N, device=dev)
    s_out = torch.empty_like(s_mid)
    stream = torch.cuda.current_stream(dev)

    def fn():
        lib7.rwkv7_wkv_prefill_bf16_path(lib7.RWKV7_PATH_AUTO, *[parts[0][n] for n in OPS], None, y[0], s_mid, stream)
        lib7.rwkv7_wkv_prefill_bf16_path(lib7.RWKV7_PATH_AUTO, *[parts[1][n] for n in OPS], s_mid, y[1], s_out,
                                         stream)

    ms = time_calls(fn, steps, stream)
    st = lib7.rwkv7_get_last_error()
    byts = prefill_bytes(B * half, H, B, state_in=False) + prefill_bytes(B * half, H, B, state_in=True)
    out = {"B": B, "T": case.T, "H": H, "calls_per_step": 2, "step_ms": ms, "tokens_per_s": B * case.T / (ms / 1e3),
           "status": st, "roofline": hbm_roofline(byts / 2, ms / 2, peaks, note="per call: half the step's bytes "
                                                   "over half the step time")}
    del parts, y, s_mid, s_out
    free_device()
    return out


def bench_ragged(lib7, dev, steps, peaks):
    """The 7.2B-width ragged batch: B=4 rows of T_b ~ U{1024..16384} tokens in packed layout, one
    varlen call."""
    case = wi.CASES[HEADLINE]
    lengths = wi.ragged_lengths(case.B, RAGGED_LO, RAGGED_HI, seed=case.seed + 11)
    d = wi.draw_packed(lengths, case.H, seed=case.seed + 12, dtype="bf16", z_mean=case.z_mean, device=dev,
                       f32_copies=False)
    dd = {n: d[n] for n in OPS}
    cu = d["cu_seqlens"].to(dev)
    total = int(lengths.sum())
    y = torch.empty_like(dd["r"])
    s_out = torch.empty(case.B, case.H, N, N, device=dev)
    stream = torch.cuda.current_stream(dev)
    max_T = int(lengths.max())

    def fn():
        lib7.rwkv7_wkv_prefill_varlen_bf16(lib7.RWKV7_PATH_AUTO, cu, max_T, *[dd[n] for n in OPS], None, y, s_out,
                                           stream)

    ms = time_calls(fn, steps, stream)
    st = lib7.rwkv7_get_last_error()
    byts = prefill_bytes(total, case.H, case.B, state_in=False)
    out = {"B": case.B, "lengths": [int(x) for x in lengths], "H": case.H, "launch_ms": ms,
           "tokens_per_s": total / (ms / 1e3), "status": st, "roofline": hbm_roofline(byts, ms, peaks)}
    del d, dd, y, s_out, cu
    free_device()
    return out


def decode_tokens(B, T, H, seed, dev, native=False):
    """Per-step token operands [T, B, H, N] (contiguous per step) drawn on the device."""
    if native:
        d = wi.draw_model_native(B, T, H, seed=seed, device=dev)
        names = NATIVE
    else:
        d = wi.draw(B, T, H, seed=seed, dtype="bf16", device=dev, f32_copies=False)
        names = OPS
    toks = {n: d[n].transpose(0, 1).contiguous() for n in names}
    extra = {"k_k": d["k_k"]} if native else {}
    del d
    return toks, extra


def bench_decode(lib7, dev, peaks, steps_target=1024, layers=24, bf16_state=False, toks=None, independent=False):
    """Decode steps/s at the L24-D1024 shape (B=256, H=16): every step reads a fresh token (1024 distinct
    tokens per CUDA graph of 1024 steps) and one of `layers` distinct states (1.6 GB in float32),
    so neither the operands nor the state stay in L2.  `bf16_state`: the state stored as bfloat16.
    `independent`: the steps set the `independent_state` option (each layer has its own state, so a
    step's state loads may start before the step before it has finished)."""
    case = wi.CASES["decode_l24_d1024_b256_1024steps"]
    B, H, T = case.B, case.H, case.T
    if toks is None:
        toks, _ = decode_tokens(B, T, H, case.seed, dev)
    states = torch.zeros(layers, B, H, N, N, device=dev, dtype=torch.bfloat16 if bf16_state else torch.float32)
    ys = [torch.empty(B, H, N, dtype=torch.bfloat16, device=dev) for _ in range(layers)]
    step_fn = lib7.rwkv7_wkv_decode_bf16_bf16state if bf16_state else lib7.rwkv7_wkv_decode_bf16
    if independent:
        ext = lib7.rwkv7_wkv_decode_ext_bf16state if bf16_state else lib7.rwkv7_wkv_decode_ext_bf16

        def step_fn(*args):
            ext(*args, independent_state=True)

    def one_pass():
        for i in range(T):
            L = i % layers
            step_fn(*[toks[n][i] for n in OPS], states[L], ys[L])

    s = torch.cuda.Stream(device=dev)
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        one_pass()  # warm-up outside the graph
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        one_pass()
    reps = max(1, math.ceil(steps_target / T))
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    st = lib7.rwkv7_get_last_error()
    ms = e0.elapsed_time(e1)
    nsteps = reps * T
    step_s = ms / 1e3 / nsteps
    byts = decode_bytes(B, H, state_elem=2 if bf16_state else 4)
    del g, states, ys
    free_device()
    out = {"B": B, "H": H, "steps": nsteps, "layer_states": layers, "state_dtype": "bf16" if bf16_state else "f32",
           "independent_state": bool(independent),
           "tokens": "fresh token every step (1024 distinct per graph)", "steps_per_s": 1.0 / step_s,
           "tokens_per_s": B / step_s, "us_per_step": step_s * 1e6, "status": st,
           "roofline": hbm_roofline(byts, step_s * 1e3, peaks)}
    if layers == 1:
        out["roofline"]["note"] = ("one state (64 MiB float32) stays in the 126 MB L2: an L2-assisted figure, "
                                   "not an HBM one")
    return out


def bench_options(lib7, dev, steps, peaks, *, native, group_norm, decode=True, layers=24):
    """The option entry points on the 0.1B prefill shape and the L24-D1024 decode shape -- model-native
    inputs (operand prologue in the kernels) and / or the ln_x GroupNorm epilogue: prefill launch time
    and HBM roofline (input tensors + y + state in and out), decode steps/s (fresh token every step)."""
    case = wi.CASES[SMALL]
    B, T, H = case.B, case.T, case.H
    names = NATIVE if native else OPS
    if native:
        d = wi.draw_model_native(B, T, H, seed=case.seed, s0_std=case.s0_std, device=dev)
    else:
        d = wi.draw(B, T, H, seed=case.seed, s0_std=case.s0_std, device=dev, f32_copies=False)
    dd = {n: d[n] for n in names}
    kk = d["k_k"] if native else None
    ln = {k: t.to(dev) for k, t in wi.draw_group_norm(H, seed=case.seed + 1).items()} if group_norm else {}
    opt = dict(model_native=native, k_k=kk, group_norm=group_norm, ln_w=ln.get("ln_w"), ln_b=ln.get("ln_b"))
    s0 = d["s0"]
    y = torch.empty(B, T, H, N, dtype=torch.bfloat16, device=dev)
    s_out = torch.empty_like(s0)
    stream = torch.cuda.current_stream(dev)

    def ops(src):
        return [src[n] for n in names] + ([None] if native else [])

    def step():
        lib7.rwkv7_wkv_prefill_ext_bf16(lib7.RWKV7_PATH_AUTO, *ops(dd), s0, y, s_out, stream=stream, **opt)

    ms = time_calls(step, steps, stream, warmup=5)
    assert lib7.rwkv7_get_last_error() == 0
    byts = prefill_bytes(B * T, H, B, n_ops=len(names))
    out = {"prefill": {"workload": SMALL, "launch_ms": ms, "tokens_per_s": B * T / (ms / 1e3),
                       "roofline": hbm_roofline(byts, ms, peaks)}}
    del d, dd, y, s_out, s0
    free_device()
    if decode:
        dc = wi.CASES["decode_l24_d1024_b256_1024steps"]
        Bd, Hd, Td = dc.B, dc.H, dc.T
        toks, extra = decode_tokens(Bd, Td, Hd, dc.seed, dev, native=native)
        dopt = dict(opt, k_k=extra.get("k_k"))
        if group_norm:
            lnd = wi.draw_group_norm(Hd, seed=dc.seed + 1)
            dopt.update(ln_w=lnd["ln_w"].to(dev), ln_b=lnd["ln_b"].to(dev))
        states = torch.zeros(layers, Bd, Hd, N, N, device=dev)
        ys = [torch.empty(Bd, Hd, N, dtype=torch.bfloat16, device=dev) for _ in range(layers)]

        def time_steps(independent):
            def one_pass():
                for i in range(Td):
                    src = {n: toks[n][i] for n in names}
                    lib7.rwkv7_wkv_decode_ext_bf16(*ops(src), states[i % layers], ys[i % layers],
                                                   independent_state=independent, **dopt)

            sd = torch.cuda.Stream(device=dev)
            sd.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(sd):
                one_pass()
            torch.cuda.current_stream().wait_stream(sd)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                one_pass()
            for _ in range(3):
                g.replay()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            g.replay()
            e1.record()
            torch.cuda.synchronize()
            assert lib7.rwkv7_get_last_error() == 0
            del g
            step_s = e0.elapsed_time(e1) / 1e3 / Td
            dbytes = decode_bytes(Bd, Hd, n_ops=len(names))
            return {"workload": "decode_l24_d1024_b256", "steps_per_s": 1.0 / step_s, "us_per_step": step_s * 1e6,
                    "tokens": "fresh token every step", "independent_state": independent,
                    "roofline": hbm_roofline(dbytes, step_s * 1e3, peaks)}

        out["decode"] = time_steps(False)
        out["decode_independent_state"] = time_steps(True)
        del toks, states, ys
        free_device()
    out["inputs"] = (("bf16 r, x_w, k, v, x_a [B,T,H,64] + float32 k_k [H,64]; w, a, b formed in-kernel"
                      if native else "bf16 r, w, k, v, a, b [B,T,H,64]")
                     + ("; y through the ln_x GroupNorm (float32 ln_w, ln_b [H,64])" if group_norm else ""))
    return out


def bench_backward(lib7, dev, peaks, steps=5, T=None):
    """The training pair on the 0.1B prefill shape: the checkpointing forward (a saved state every 64
    tokens) and the backward (float32 gradients of r, w, k, v, a, b and the initial state).
    Reports ms per call, tokens/s and each call's HBM roofline; the backward is bound by its per-token
    CUDA-core work (its fraction of HBM shows how far from the memory bound that leaves it)."""
    case = wi.CASES[SMALL]
    B, H = case.B, case.H
    T = T or case.T
    d = wi.draw(B, T, H, seed=case.seed, s0_std=case.s0_std, device=dev, f32_copies=False)
    gr = wi.draw_grads(B, T, H, seed=case.seed + 2)
    dd = {n: d[n] for n in OPS}
    s0 = d["s0"]
    dy, ds = gr["dy"].to(dev), gr["ds_out"].to(dev)
    y = torch.empty_like(dd["r"])
    s_out = torch.empty_like(s0)
    states = torch.empty((B, H, lib7.n_checkpoints(T), N, N), dtype=torch.float32, device=dev)
    g = [torch.empty((B, T, H, N), dtype=torch.float32, device=dev) for _ in range(6)]
    ds_in = torch.empty_like(s0)
    stream = torch.cuda.current_stream(dev)

    def fwd():
        lib7.rwkv7_wkv_prefill_save_bf16(*[dd[n] for n in OPS], s0, y, s_out, states, stream)

    def bwd():
        lib7.rwkv7_wkv_backward_bf16(*[dd[n] for n in OPS], states, dy, ds, *g, ds_in, stream)

    out = {}
    nbytes = dict(zip(("forward_save", "backward"), training_bytes(B, T, H)))
    for name, fn in (("forward_save", fwd), ("backward", bwd)):
        ms = time_calls(fn, steps, stream, warmup=2)
        out[name] = {"ms": ms, "tokens_per_s": B * T / (ms / 1e3), "roofline": hbm_roofline(nbytes[name], ms, peaks)}
    assert lib7.rwkv7_get_last_error() == 0
    out["workload"] = SMALL if T == case.T else f"{SMALL} at T={T}"
    out["outputs"] = "float32 dr, dw, dk, dv, da, db [B,T,H,64] and ds_in; dy bf16, ds_out float32"
    del d, dd, y, s_out, states, g
    free_device()
    return out


# ---- our arm ------------------------------------------------------------------------------------------

SCHEDULES = {"auto": 0, "pair": 1, "tasks": 2, "pipe": 3}


def run_ours(args):
    world, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    import rwkv_delta_rule_b200 as lib7

    lib7.load_library()
    peaks, peak_kind = load_peaks()
    case = wi.CASES[HEADLINE]
    B = args.batch or case.B
    T = args.seqlen or case.T
    H = case.H
    from rwkv_delta_rule_b200.dist import rank_seed

    d = wi.draw(B, T, H, seed=rank_seed(case.seed, rank), dtype="bf16", z_mean=case.z_mean, s0_std=case.s0_std,
                device=dev, f32_copies=False)
    dd = {n: d[n] for n in OPS}
    s0 = d["s0"]
    y = torch.empty_like(dd["r"])
    s_out = torch.empty(B, H, N, N, device=dev)
    sched = SCHEDULES[args.schedule]
    stream = torch.cuda.current_stream(dev)

    if sched:
        def step():
            lib7.rwkv7_wkv_prefill_ext_bf16(lib7.RWKV7_PATH_CHUNK, *[dd[n] for n in OPS], s0, y, s_out,
                                            schedule=sched, stream=stream)
    else:
        def step():
            lib7.rwkv7_wkv_prefill_bf16_path(lib7.RWKV7_PATH_AUTO, *[dd[n] for n in OPS], s0, y, s_out, stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert lib7.rwkv7_get_last_error() == 0

    # per-launch durations over the timed region, on the launching stream
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    e_start, e_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local, args.clocks_csv)
    with clocks:
        barrier(world)
        torch.cuda.synchronize()
        e_start.record(stream)
        for i in range(args.steps):
            evs[i][0].record(stream)
            step()
            evs[i][1].record(stream)
        e_stop.record(stream)
        torch.cuda.synchronize()
        barrier(world)
    ms_total = max_over_ranks(e_start.elapsed_time(e_stop), world)
    per_launch_ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
    assert lib7.rwkv7_get_last_error() == 0

    tokens_per_step = B * T * world
    value = tokens_per_step * args.steps / (ms_total / 1e3)

    e2e = None
    if not args.no_e2e:
        # end to end through the C ABI with host buffers (inputs copied once to pinned host memory
        # before the timed region; every timed call copies them up and the results back)
        host = {n: dd[n].cpu().pin_memory() for n in OPS}
        host_s0 = s0.cpu().pin_memory() if s0 is not None else None
        host_y = torch.empty(y.shape, dtype=y.dtype).pin_memory()
        host_s = torch.empty(s_out.shape, dtype=torch.float32).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        h2d += host_s0.numel() * 4 if host_s0 is not None else 0
        d2h = host_y.numel() * host_y.element_size() + host_s.numel() * 4
        staging = {**dd, "s_in": s0, "y": y, "s_out": s_out}

        def e2e_step():
            lib7.rwkv7_wkv_prefill_host_bf16(lib7.RWKV7_PATH_AUTO, *[host[n] for n in OPS], host_s0, host_y, host_s,
                                             staging, slices=args.e2e_slices, stream=stream)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        k_e2e = max(3, min(args.steps, args.e2e_steps))
        barrier(world)
        torch.cuda.synchronize()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(k_e2e):
            e2e_step()
        a1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        assert lib7.rwkv7_get_last_error() == 0
        e2e_ms = max_over_ranks(a0.elapsed_time(a1), world)
        e2e = {"value": tokens_per_step * k_e2e / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "steps": k_e2e, "call": "rwkv7_wkv_prefill_host_bf16",
               "slices": args.e2e_slices or "auto"}
        del host, host_s0, host_y, host_s, staging

    algo = prefill_bytes(B * T, H, B, state_in=s0 is not None)
    roofline = hbm_roofline(algo, per_launch_ms, peaks, traffic=(args.traffic if args.traffic is not None
                                                                 else measured_traffic(B, T, H, args.schedule)),
                            peak_source=peak_kind, kernel="wkv7 chunked prefill (tcgen05)",
                            peak_kind="burst copy bandwidth (kernel timed back to back, about 3 ms per launch)",
                            tensor_view=tensor_view(B * T, H, per_launch_ms, peaks))
    del d, dd, y, s_out, s0
    free_device()

    per_workload = None
    schedules = None
    if not args.no_configs:
        K = args.config_steps
        per_workload = {"prefill_f32_b1_t64_h2": bench_f32_small(lib7, dev, 200, peaks),
                   "prefill_d768_b8_t4096": bench_prefill(lib7, dev, SMALL, K, peaks),
                   "prefill_d2048_b16_t8192_chained": bench_chained(lib7, dev, K, peaks)}
        if not args.no_decode:
            dec = bench_decode(lib7, dev, peaks, steps_target=args.decode_steps, layers=args.decode_layers)
            dec["bf16_state"] = bench_decode(lib7, dev, peaks, steps_target=args.decode_steps,
                                             layers=args.decode_layers, bf16_state=True)
            dec["l2_assisted_single_state"] = bench_decode(lib7, dev, peaks, steps_target=args.decode_steps, layers=1)
            # the same steps with the independent_state option (the 24 layer states are distinct, so a step's
            # state loads may overlap the last wave of the step before)
            dec["independent_state"] = bench_decode(lib7, dev, peaks, steps_target=args.decode_steps,
                                                    layers=args.decode_layers, independent=True)
            dec["bf16_state_independent_state"] = bench_decode(lib7, dev, peaks, steps_target=args.decode_steps,
                                                               layers=args.decode_layers, bf16_state=True,
                                                               independent=True)
            per_workload["decode_l24_d1024_b256_1024steps"] = dec
        per_workload[HEADLINE] = {"B": B, "T": T, "H": H, "launch_ms": per_launch_ms,
                             "tokens_per_s": B * T / (per_launch_ms / 1e3), "status": 0, "roofline": roofline,
                             "note": "the headline step"}
        per_workload["prefill_d4096_b4_ragged"] = bench_ragged(lib7, dev, K, peaks)
        schedules = {"pipelined (schedule 3)": {
            SMALL: bench_prefill(lib7, dev, SMALL, K, peaks, schedule=3),
            HEADLINE: bench_prefill(lib7, dev, HEADLINE, max(3, K // 2), peaks, schedule=3)}}

    native = None
    if not args.no_native:
        native = {key: bench_options(lib7, dev, min(args.steps, 50), peaks, native=nat, group_norm=gn,
                                     decode=not args.no_decode)
                  for key, nat, gn in (("model_native", True, False), ("group_norm", False, True),
                                       ("model_native_group_norm", True, True))}

    train = None
    if not args.no_backward:
        train = bench_backward(lib7, dev, peaks, T=args.train_seqlen or None)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        T_s = min(case.T, args.ref_tokens)
        v, reps, el, threads = time_oracle(oracle_sample(T_s, device=dev), args.cpu_budget)
        cpu = {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle",
               "sample": f"batch row 0 of {case.B} (all {H} heads) x first {T_s} of {case.T} tokens, {reps} rep(s), "
                         f"{el:.1f} s, float64 C oracle on {threads} threads ({cpu_model()})"}

    line = {
        "metric": "wkv7 prefill tokens/s", "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": HEADLINE, "B": B, "T": T, "H": H, "N": N, "global_batch": B * world, "seq_len": T,
                   "parallelism": f"replicas x{world} (batch-sharded, no exchange)",
                   "l2": f"operands larger than L2 ({algo / 1e6:.0f} MB per step vs 126 MB); no flush",
                   "schedule": args.schedule, "state": "float32 out (zero initial state)",
                   "inputs": "bf16 r, w, k, v, a, b; w from z ~ N(1, 1)"},
        "e2e": e2e,
        "roofline": roofline,
        "gpu_launches": args.steps,
        "clocks": clocks.summary(),
        "cpu_baseline": cpu,
        "configs": per_workload,
        "schedules": schedules,
        "options": native,
        "training": train,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--schedule", choices=tuple(SCHEDULES), default="auto",
                    help="chunk schedule of the headline prefill (auto: the library's choice)")
    ap.add_argument("--batch", type=int, default=0, help="override B of the headline (profiling runs only)")
    ap.add_argument("--seqlen", type=int, default=0, help="override T of the headline (profiling runs only)")
    ap.add_argument("--no-configs", action="store_true", help="skip the per-workload table")
    ap.add_argument("--config-steps", type=int, default=20)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-native", action="store_true",
                    help="skip the option entry points' lines (model-native inputs, GroupNorm epilogue)")
    ap.add_argument("--no-backward", action="store_true", help="skip the training (forward-save + backward) line")
    ap.add_argument("--train-seqlen", type=int, default=0, help="override T of the training leg (profiling runs only)")
    ap.add_argument("--decode-steps", type=int, default=3072)
    ap.add_argument("--decode-layers", type=int, default=24, help="distinct decode states rotated over")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--clocks-csv", default=None, help="also write the raw nvidia-smi clock samples here")
    ap.add_argument("--e2e-slices", type=int, default=0,
                    help="batch slices of the host-buffer call in the e2e leg (0: chosen by the library)")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    ap.add_argument("--ref-tokens", type=int, default=4096)
    ap.add_argument("--traffic", type=float, default=None,
                    help="ncu dram bytes per launch of the prefill kernel, if captured for this build")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
