#!/usr/bin/env python
"""Throughput benchmark of the RWKV-7 (x070) state-recurrence library on B200.

A step is one prefill call over one batch of the 0.1B-shaped workload
(D768: B=8 sequences x T=4096 tokens x H=12 heads of size 64, bf16 operands,
float32 state carried in and out), which is the workload the headline metric
is quoted on.  The prefill kernel reads the six operand tensors and writes y
and the final state: 355.5 MB per step, larger than the 126 MB L2, so no L2
flush is needed between steps.

One JSON line is printed by rank 0:
  value      prefill tokens/s over all ranks (device time, CUDA events, max over ranks)
  e2e        the same metric through the C-ABI call with host buffers
             (rwkv7_wkv_prefill_host_bf16): pinned host -> device copies of the
             operands and initial state, the prefill, and device -> host copies of
             y and the final state, in batch slices whose copies overlap the
             compute of other slices; all timed
  roofline   the prefill kernel's algorithmic HBM bytes / its average launch time
  decode     wkv7s decode steps/s at the L24-D1024 shape (B=256, H=16), rotating
             over 24 layer states (1.6 GB) so the state cannot stay in L2
  cpu_baseline  the float64 oracle on this host's cores (rank 0, N=1 only)

Multi-GPU (torchrun): every rank runs its own batch (weak scaling); the
recurrence has no cross-rank exchange, so the only collectives are the
barrier and the max-reduction of the timings.

``--impl reference`` times the float64 CPU oracle instead (the only other
program this workload has), on rank 0, on the same workload and metric.
"""

from __future__ import annotations

import argparse
import json
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
WORKLOAD = "prefill_d768_b8_t4096"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one chunk-kernel launch, from one ncu
# capture at B=4 (48 pairs on the task-parallel schedule, as at B=8; 178 MB of operands, larger than
# L2) scaled by B to the B=8 workload; the
# figure holds only for the kernel source it was taken on (sha256 prefix of wkv7_chunk.cu), and the
# line reports null for any other build.  The capture is summarised under profiles/.
MEASURED_TRAFFIC = {"source_sha256": "e56f7e438c3e1b20", "bytes_per_token_head": (151925760 + 14336768) / (4 * 4096 * 12)}


def measured_traffic(B, T, H, path):
    import hashlib
    src = os.path.join(ROOT, "rwkv_delta_rule_b200", "csrc", "wkv7_chunk.cu")
    try:
        with open(src, "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()[:16]
    except OSError:
        return None
    if sha != MEASURED_TRAFFIC["source_sha256"] or path == "scan":
        return None
    return MEASURED_TRAFFIC["bytes_per_token_head"] * B * T * H


def prefill_bytes(B, T, H, elem=2):
    """Algorithmic HBM bytes of one prefill call: six operands read, y written
    (B*T*H*N elements each) and the state read and written (B*H*N*N float32)."""
    return 7 * B * T * H * N * elem + 2 * B * H * N * N * 4


def decode_bytes(B, H, elem=2):
    """Algorithmic HBM bytes of one decode step: state read + written, six
    operand vectors read, y written."""
    return B * H * (2 * N * N * 4 + 7 * N * elem)


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


# ---- CPU oracle timing -------------------------------------------------------------------------------

def time_oracle(d, B, T, H, budget_s: float, min_reps: int = 1):
    """Run the float64 oracle over the whole workload (all pairs, all tokens)
    until about `budget_s` seconds have passed; returns (tokens/s, reps, seconds, threads)."""
    import oracle

    ops = [d[n + "_f32"] for n in OPS]
    threads = oracle.default_threads()
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle.wkv7(*ops, d["s0"], nthreads=threads)
        reps += 1
        el = time.perf_counter() - t0
        if reps >= min_reps and el >= budget_s:
            break
        if reps >= min_reps and el * (reps + 1) / reps > budget_s * 3:
            break
    return B * T * reps / el, reps, el, threads


def time_oracle_sample(d, B, T, H, T_sample: int, budget_s: float):
    """Oracle on the first T_sample tokens of every (b, h) pair (bounded sample)."""
    sub = {n + "_f32": d[n + "_f32"][:, :T_sample] for n in OPS}
    sub["s0"] = d["s0"]
    return time_oracle(sub, B, T_sample, H, budget_s)


# ---- reference arm ------------------------------------------------------------------------------------

def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    case = wi.CASES[WORKLOAD]
    d = wi.draw_case(case)
    import oracle

    threads = oracle.default_threads()
    T_sample = min(case.T, args.ref_tokens)
    sub = [d[n + "_f32"][:, :T_sample] for n in OPS]
    for _ in range(args.warmup):
        oracle.wkv7(*sub, d["s0"], nthreads=threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.wkv7(*sub, d["s0"], nthreads=threads)
    el = time.perf_counter() - t0
    value = case.B * T_sample * args.steps / el
    sample = (f"all {case.B * case.H} (b,h) pairs x first {T_sample} of {case.T} tokens per step, "
              f"float64 C oracle, {threads} threads")
    line = {
        "impl": "reference", "metric": "wkv7 prefill tokens/s", "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "B": case.B, "T": case.T, "H": case.H, "N": N, "global_batch": case.B,
                   "seq_len": case.T, "parallelism": "replicas only", "operands": "bf16 (exact in fp64)"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---- our arm ------------------------------------------------------------------------------------------

def bench_decode(lib7, dev, steps_target: int = 1024, layers: int = 24, bf16_state: bool = False):
    """Decode steps/s at B=256, H=16, rotating over `layers` distinct states (bf16_state: the
    reduced-precision variant whose state is stored as bfloat16)."""
    case = wi.CASES["decode_l24_d1024_b256_1024steps"]
    B, H = case.B, case.H
    ntok = 8
    d = wi.draw(B, ntok, H, seed=case.seed, dtype="bf16")
    toks = [{n: d[n][:, t].contiguous().to(dev) for n in OPS} for t in range(ntok)]
    states = torch.zeros(layers, B, H, N, N, device=dev, dtype=torch.bfloat16 if bf16_state else torch.float32)
    ys = [torch.empty(B, H, N, dtype=torch.bfloat16, device=dev) for _ in range(layers)]
    per_graph = layers * 4
    step_fn = lib7.rwkv7_wkv_decode_bf16_bf16state if bf16_state else lib7.rwkv7_wkv_decode_bf16

    def one_pass(start):
        for i in range(per_graph):
            L = (start + i) % layers
            tk = toks[(start + i) % ntok]
            step_fn(*[tk[n] for n in OPS], states[L], ys[L])

    s = torch.cuda.Stream(device=dev)
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        one_pass(0)  # warm-up outside the graph
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        one_pass(0)
    reps = max(1, (steps_target + per_graph - 1) // per_graph)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    nsteps = reps * per_graph
    step_s = ms / 1e3 / nsteps
    byts = decode_bytes(B, H) - (B * H * 2 * N * N * 2 if bf16_state else 0)
    return {"workload": "decode_l24_d1024_b256", "B": B, "H": H, "steps": nsteps, "layer_states": layers,
            "state_dtype": "bf16" if bf16_state else "f32",
            "state_bytes_total": layers * B * H * N * N * (2 if bf16_state else 4), "steps_per_s": 1.0 / step_s,
            "tokens_per_s": B / step_s, "us_per_step": step_s * 1e6, "bytes_per_step": byts,
            "achieved_gbs": byts / step_s / 1e9, "launches": nsteps}


NATIVE = ("r", "xw", "k", "v", "xa")


def bench_options(lib7, dev, B, T, H, steps, *, native, group_norm, decode_steps=1024, layers=24):
    """The option entry points on the same shapes -- model-native inputs (operand prologue in the
    kernels) and / or the ln_x GroupNorm epilogue: prefill launch time and HBM roofline (input tensors
    + y + state in and out), and decode steps/s at the L24-D1024 shape."""
    case = wi.CASES[WORKLOAD]
    names = NATIVE if native else OPS
    d = (wi.draw_model_native if native else wi.draw)(B, T, H, seed=case.seed, s0_std=case.s0_std)
    dd = {n: d[n].to(dev) for n in names}
    kk = d["k_k"].to(dev) if native else None
    ln = {k: t.to(dev) for k, t in wi.draw_group_norm(H, seed=case.seed + 1).items()} if group_norm else {}
    opt = dict(model_native=native, k_k=kk, group_norm=group_norm, ln_w=ln.get("ln_w"), ln_b=ln.get("ln_b"))
    s0 = d["s0"].to(dev)
    y = torch.empty_like(dd["r"])
    s_out = torch.empty_like(s0)
    stream = torch.cuda.current_stream(dev)

    def ops(src):
        return [src[n] for n in names] + ([None] if native else [])

    def step():
        lib7.rwkv7_wkv_prefill_ext_bf16(lib7.RWKV7_PATH_AUTO, *ops(dd), s0, y, s_out, stream=stream, **opt)

    for _ in range(5):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    assert lib7.rwkv7_get_last_error() == 0
    ms = e0.elapsed_time(e1) / steps
    byts = (len(names) + 1) * B * T * H * N * 2 + 2 * B * H * N * N * 4
    peaks, _ = load_peaks()
    pre = {"launch_ms": ms, "tokens_per_s": B * T / (ms / 1e3), "algorithmic_bytes_per_launch": byts,
           "achieved_gbs": byts / (ms / 1e3) / 1e9, "frac": byts / (ms / 1e3) / 1e9 / peaks["hbm_gbs"]}
    del dd, y, s_out
    out = {"prefill": pre}
    if decode_steps:
        dc = wi.CASES["decode_l24_d1024_b256_1024steps"]
        Bd, Hd, ntok = dc.B, dc.H, 8
        dn = (wi.draw_model_native if native else wi.draw)(Bd, ntok, Hd, seed=dc.seed)
        toks = [{n: dn[n][:, t].contiguous().to(dev) for n in names} for t in range(ntok)]
        dopt = dict(opt, k_k=dn["k_k"].to(dev) if native else None)
        if group_norm:
            lnd = wi.draw_group_norm(Hd, seed=dc.seed + 1)
            dopt.update(ln_w=lnd["ln_w"].to(dev), ln_b=lnd["ln_b"].to(dev))
        states = torch.zeros(layers, Bd, Hd, N, N, device=dev)
        ys = [torch.empty(Bd, Hd, N, dtype=torch.bfloat16, device=dev) for _ in range(layers)]
        per_graph = layers * 4

        def one_pass():
            for i in range(per_graph):
                lib7.rwkv7_wkv_decode_ext_bf16(*ops(toks[i % ntok]), states[i % layers], ys[i % layers], **dopt)

        sd = torch.cuda.Stream(device=dev)
        sd.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(sd):
            one_pass()
        torch.cuda.current_stream().wait_stream(sd)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            one_pass()
        reps = max(1, (decode_steps + per_graph - 1) // per_graph)
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        e0.record()
        for _ in range(reps):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        assert lib7.rwkv7_get_last_error() == 0
        step_s = e0.elapsed_time(e1) / 1e3 / (reps * per_graph)
        dbytes = Bd * Hd * (2 * N * N * 4 + (len(names) + 1) * N * 2)
        out["decode"] = {"workload": "decode_l24_d1024_b256", "steps_per_s": 1.0 / step_s,
                         "us_per_step": step_s * 1e6, "bytes_per_step": dbytes, "achieved_gbs": dbytes / step_s / 1e9,
                         "frac": dbytes / step_s / 1e9 / peaks["hbm_gbs"]}
    out["inputs"] = (("bf16 r, x_w, k, v, x_a [B,T,H,64] + float32 k_k [H,64]; w, a, b formed in-kernel"
                      if native else "bf16 r, w, k, v, a, b [B,T,H,64]")
                     + ("; y through the ln_x GroupNorm (float32 ln_w, ln_b [H,64])" if group_norm else ""))
    return out


def bench_backward(lib7, dev, B, T, H, steps=5):
    """The training pair on the same shapes: the checkpointing forward (scan with a saved state every
    64 tokens) and the backward (float32 gradients of r, w, k, v, a, b and the initial state).
    Reports ms per call and tokens/s; the backward is bound by its per-token CUDA-core work."""
    case = wi.CASES[WORKLOAD]
    d = wi.draw(B, T, H, seed=case.seed, s0_std=case.s0_std)
    gr = wi.draw_grads(B, T, H, seed=case.seed + 2)
    dd = {n: d[n].to(dev) for n in OPS}
    s0 = d["s0"].to(dev)
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
    for name, fn in (("forward_save", fwd), ("backward", bwd)):
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / steps
        out[name] = {"ms": ms, "tokens_per_s": B * T / (ms / 1e3)}
    assert lib7.rwkv7_get_last_error() == 0
    out["workload"] = WORKLOAD
    out["outputs"] = "float32 dr, dw, dk, dv, da, db [B,T,H,64] and ds_in; dy bf16, ds_out float32"
    return out


def run_ours(args):
    world, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    import rwkv_delta_rule_b200 as lib7

    lib7.load_library()
    case = wi.CASES[WORKLOAD]
    B = args.batch or case.B
    T = args.seqlen or case.T
    H = case.H
    from rwkv_delta_rule_b200.dist import rank_seed

    d = wi.draw(B, T, H, seed=rank_seed(case.seed, rank), dtype="bf16", s0_std=case.s0_std)
    dd = {n: d[n].to(dev) for n in OPS}
    s0 = d["s0"].to(dev)
    y = torch.empty_like(dd["r"])
    s_out = torch.empty_like(s0)
    path = {"auto": lib7.RWKV7_PATH_AUTO, "scan": lib7.RWKV7_PATH_SCAN, "chunk": lib7.RWKV7_PATH_CHUNK}[args.path]
    stream = torch.cuda.current_stream(dev)

    def step():
        lib7.rwkv7_wkv_prefill_bf16_path(path, *[dd[n] for n in OPS], s0, y, s_out, stream)

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
        # end to end through the C ABI with host buffers
        host = {n: d[n].pin_memory() for n in OPS}
        host_s0 = d["s0"].pin_memory()
        host_y = torch.empty(y.shape, dtype=y.dtype).pin_memory()
        host_s = torch.empty(s_out.shape, dtype=torch.float32).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in host.values()) + host_s0.numel() * 4
        d2h = host_y.numel() * host_y.element_size() + host_s.numel() * 4

        staging = {**dd, "s_in": s0, "y": y, "s_out": s_out}

        def e2e_step():
            # one C-ABI call: per batch slice, pinned host -> device copies of the operands and the
            # initial state, the prefill, and device -> host copies of y and the final state, the
            # copies of one slice overlapping the compute and copies of others
            lib7.rwkv7_wkv_prefill_host_bf16(path, *[host[n] for n in OPS], host_s0, host_y, host_s, staging,
                                             slices=args.e2e_slices, stream=stream)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        k_e2e = max(3, min(args.steps, 20))
        barrier(world)
        torch.cuda.synchronize()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(k_e2e):
            e2e_step()
        a1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        e2e_ms = max_over_ranks(a0.elapsed_time(a1), world)
        e2e_value = tokens_per_step * k_e2e / (e2e_ms / 1e3)
        e2e = {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "steps": k_e2e, "call": "rwkv7_wkv_prefill_host_bf16", "slices": args.e2e_slices or "auto"}

    peaks, peak_kind = load_peaks()
    algo = prefill_bytes(B, T, H)
    achieved = algo / (per_launch_ms / 1e3) / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"],
                "traffic": args.traffic if args.traffic is not None else measured_traffic(B, T, H, args.path),
                "peak_source": peak_kind,
                "kernel": "prefill", "algorithmic_bytes_per_launch": algo, "launch_ms": per_launch_ms}

    decode = None
    if not args.no_decode:
        decode = bench_decode(lib7, dev, steps_target=args.decode_steps, layers=args.decode_layers)
        decode["frac"] = decode["achieved_gbs"] / peaks["hbm_gbs"]
        assert lib7.rwkv7_get_last_error() == 0
        d16 = bench_decode(lib7, dev, steps_target=args.decode_steps, layers=args.decode_layers, bf16_state=True)
        d16["frac"] = d16["achieved_gbs"] / peaks["hbm_gbs"]
        assert lib7.rwkv7_get_last_error() == 0
        decode["bf16_state"] = {k: d16[k] for k in ("state_dtype", "steps_per_s", "tokens_per_s", "us_per_step",
                                                    "bytes_per_step", "achieved_gbs", "frac")}

    native = None
    if not args.no_native and args.path == "auto":
        native = {key: bench_options(lib7, dev, B, T, H, steps=min(args.steps, 50), native=nat, group_norm=gn,
                                     decode_steps=0 if args.no_decode else args.decode_steps)
                  for key, nat, gn in (("model_native", True, False), ("group_norm", False, True),
                                       ("model_native_group_norm", True, True))}

    train = None
    if not args.no_backward and args.path == "auto":
        train = bench_backward(lib7, dev, B, T, H)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        T_s = min(T, args.ref_tokens)
        v, reps, el, threads = time_oracle_sample(d, B, T, H, T_s, args.cpu_budget)
        cpu = {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle",
               "sample": f"all {B * H} (b,h) pairs x first {T_s} of {T} tokens, {reps} rep(s), {el:.1f} s, "
                         f"float64 C oracle"}

    launches_per_step = 1
    line = {
        "metric": "wkv7 prefill tokens/s", "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "B": B, "T": T, "H": H, "N": N, "global_batch": B * world, "seq_len": T,
                   "parallelism": f"replicas x{world} (batch-sharded, no exchange)",
                   "l2": "operands larger than L2 (355 MB per step vs 126 MB); no flush",
                   "path": args.path, "state": "float32 in/out"},
        "e2e": e2e,
        "roofline": roofline,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks.summary(),
        "cpu_baseline": cpu,
        "decode": decode,
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
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--path", choices=("auto", "scan", "chunk"), default="auto")
    ap.add_argument("--batch", type=int, default=0, help="override B (profiling runs only)")
    ap.add_argument("--seqlen", type=int, default=0, help="override T (profiling runs only)")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-native", action="store_true",
                    help="skip the option entry points' lines (model-native inputs, GroupNorm epilogue)")
    ap.add_argument("--no-backward", action="store_true", help="skip the training (forward-save + backward) line")
    ap.add_argument("--decode-steps", type=int, default=1024)
    ap.add_argument("--decode-layers", type=int, default=24, help="distinct decode states rotated over")
    ap.add_argument("--no-e2e", action="store_true")
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
