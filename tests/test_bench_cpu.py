"""CPU checks of bench.py's JSON contract on the leg that needs no GPU: the reference arm (the
float64 oracle timed on the host cores) prints one line with the base contract's keys, its own
cpu_baseline and a zero-byte e2e, on the bench's workload configuration."""

import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0"],
                         cwd=ROOT, capture_output=True, text=True, timeout=300, check=True).stdout
    lines = [ln for ln in out.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["value"] > 0 and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["config"]["workload"] == "prefill_d4096_b4_t16384"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def _bench():
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import bench

    return bench


def test_bench_algorithmic_bytes_and_flops():
    # the roofline arithmetic against the workloads' own figures: 896 B per token-head for six bf16
    # operands and y, 16 KiB per state, 33,664 B per decode head-step, 99.7 kflop per token-head at C = 64
    b = _bench()
    assert b.prefill_bytes(8 * 4096, 12, 8) == 7 * 8 * 4096 * 12 * 64 * 2 + 2 * 8 * 12 * 64 * 64 * 4 == 355467264
    assert b.prefill_bytes(4 * 16384, 64, 4, state_in=False) == 7 * 4 * 16384 * 64 * 128 + 4 * 64 * 16384
    assert b.prefill_bytes(64, 2, 1, elem=4, state_in=False) == 7 * 64 * 2 * 64 * 4 + 2 * 64 * 64 * 4
    assert b.decode_bytes(256, 16) == 256 * 16 * 33664 == 137887744
    assert b.decode_bytes(256, 16, state_elem=2) == 256 * 16 * (2 * 64 * 64 * 2 + 7 * 64 * 2)
    assert b.decode_bytes(256, 16, n_ops=5) == 256 * 16 * (2 * 64 * 64 * 4 + 6 * 64 * 2)
    assert abs(b.PREFILL_FLOP_PER_TOKEN_HEAD - 99669.33) < 0.01
    # training pair at B8 T4096 H12: per token-head 7 bf16 vectors forward (6 operands + y) and 7 bf16
    # + 6 float32 vectors backward; per pair 64 saved states plus two more (s_in/s_out, ds_out/ds_in)
    fwd, bwd = b.training_bytes(8, 4096, 12)
    assert fwd == 8 * 4096 * 12 * 896 + 96 * 66 * 16384
    assert bwd == 8 * 4096 * 12 * (896 + 1536) + 96 * 66 * 16384
    assert b.training_bytes(1, 65, 1) == (65 * 896 + 4 * 16384, 65 * 2432 + 4 * 16384)  # two chunks
    peaks = {"hbm_gbs": 1000.0, "bf16_tflops": 1000.0}
    r = b.hbm_roofline(2e9, 4.0, peaks)  # 2 GB in 4 ms = 500 GB/s
    assert abs(r["achieved"] - 500.0) < 1e-9 and abs(r["frac"] - 0.5) < 1e-12 and r["unit"] == "GB/s"
    t = b.tensor_view(1000, 10, 1.0, peaks)  # 1e4 token-heads x 99.7 kflop in 1 ms
    assert abs(t["achieved"] - 1e4 * b.PREFILL_FLOP_PER_TOKEN_HEAD / 1e-3 / 1e12) < 1e-9
    assert t["bound"] == "tensor" and abs(t["frac"] - t["achieved"] / 1000.0) < 1e-12


def test_bench_clock_summary_flags_throttling():
    b = _bench()
    c = b.ClockSampler(0)
    c.lines = ["0, 1965, 1965, 700, 0x0, Not Active, Not Active, Not Active, Not Active",
               "0, 1900, 1965, 990, 0x4, Not Active, Not Active, Not Active, Active",
               "0, 1500, 1965, 400, 0x20, Not Active, Active, Not Active, Not Active"]
    s = c.summary()
    assert s["sm_max_mhz"] == 1965.0 and s["samples"] == 3
    assert s["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]
    c.lines = []
    assert c.summary()["reasons"] == ["unsampled"]
