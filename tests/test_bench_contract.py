"""bench.py's command-line contract, on the CPU: the reference arm (the oracle on the host cores)
prints one JSON line with the keys the driver reads, the non-zero ranks of a multi-rank launch of
that arm exit 0 without work, and fewer than 3 warm-up steps are refused."""
import json
import os
import pathlib
import subprocess
import sys

ROOT = pathlib.Path(__file__).resolve().parent.parent


def run(args, env_extra=None):
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, str(ROOT / "bench.py"), *args], cwd=ROOT, env=env,
                          capture_output=True, text=True, timeout=600)


def test_reference_arm_prints_one_json_line_with_the_contract_keys():
    r = run(["--impl", "reference", "--workload", "tiny", "--steps", "3", "--warmup", "3"])
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference"
    assert d["value"] > 0 and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["steps"] == 3 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["config"]["workload"].startswith("tiny")
    # the line states what each step ran: a few fresh tokens, host-drawn weights
    assert d["config"]["T_sampled"] == 8 and "fresh tokens per step" in d["config"]["sample"]
    assert "not the GPU arm's weights" in d["config"]["expert_weights"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert set(cb["phases_s"]) == {"route", "experts", "combine"}
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_without_work():
    r = run(["--impl", "reference", "--workload", "tiny", "--steps", "3", "--warmup", "3"],
            {"RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_fewer_than_three_warmup_steps_are_refused():
    r = run(["--impl", "reference", "--workload", "tiny", "--steps", "3", "--warmup", "2"])
    assert r.returncode != 0
    assert "--warmup must be >= 3" in r.stderr


def test_cpu_baseline_batches_the_expert_rows_and_names_its_phases():
    """The GPU arm's CPU baseline, run here on the tiny workload's host tensors: every FFN pick of
    the sampled tokens goes through the oracle in calls of many rows (grouped by expert), and the
    line names the routed and FFN token counts, the per-phase times and the thread count."""
    sys.path.insert(0, str(ROOT))
    import bench
    import oracle
    from mixture_experts_zero_b200 import inputs
    w = inputs.WORKLOADS["tiny"]
    data = inputs.make(w, device="cpu")
    cb = bench.cpu_baseline(w, data, ffn_tokens=32, chunk=4)
    assert cb["value"] > 0 and cb["kind"] == "oracle"
    assert cb["cores"] == oracle.num_threads()
    assert cb["tokens"]["routed"] == w.T and cb["tokens"]["ffn"] == 32
    assert cb["tokens"]["ffn_picks"] > 0
    assert "subset-measured" in cb["sample"] and f"{cb['cores']} threads" in cb["sample"]
    # N = 8 experts in groups of 4: two oracle calls, each with the rows of four experts
    assert "2 oracle calls" in cb["sample"]


def test_cpu_baseline_of_a_whole_batch_says_so():
    """With the FFN sample as large as the batch, every token is routed and run through the
    experts: the line is labelled a full-batch measurement."""
    sys.path.insert(0, str(ROOT))
    import bench
    from mixture_experts_zero_b200 import inputs
    w = inputs.WORKLOADS["tiny"]
    cb = bench.cpu_baseline(w, inputs.make(w, device="cpu"), ffn_tokens=w.T)
    assert cb["tokens"]["routed"] == w.T and cb["tokens"]["ffn"] == w.T
    assert cb["sample"].startswith("full batch: ")


def test_control_loop_cpu_baseline_times_route_and_update():
    """The bias-control loop's CPU baseline: the oracle's router logits, routing and bias update
    on the loop's first steps, reported per control step and per token."""
    sys.path.insert(0, str(ROOT))
    import bench
    import oracle
    from mixture_experts_zero_b200 import inputs
    w = inputs.scaled(inputs.WORKLOADS["bias_loop"], T=64, d=256)
    line = bench.control_cpu_baseline(w, "cpu", steps=2)
    assert line["impl"] == "cpu_baseline" and line["kind"] == "oracle"
    assert line["cores"] == oracle.num_threads()
    assert line["control_step_ms"] > 0
    # both figures come from the same mean step time (the milliseconds rounded to 1 us)
    ms = line["control_step_ms"]
    assert abs(line["tokens_per_s"] - w.T / (ms / 1e3)) <= (0.0005 / ms + 1e-6) * line["tokens_per_s"] + 0.1
    assert "first 2 of the 200 control steps" in line["sample"]


def test_gemm_phase_roofline_splits_rows_by_tile_kind():
    """Rows per expert 0, 100, 200, 300 and 600: both GEMMs take rows into 256-row tiles from 128
    rows (200; 256 of 300 with a 44-row leftover streamed; 512 of 600 with an 88-row leftover
    streamed) and stream the 100-row expert's weights."""
    sys.path.insert(0, str(ROOT))
    import bench
    d, I = 64, 32
    counts = [0, 100, 200, 300, 600]
    r = bench.gemm_phase_roofline(counts, d, I, False, {"gemm1_swiglu": 1000.0, "gemm2_down": 1000.0},
                                  sm_count=2, hbm_gbs=1.0, measured_ms={"gemm1_swiglu": 1.0, "gemm2_down": 1.0})
    g1, g2 = r["gemm1_swiglu"], r["gemm2_down"]
    assert g1["rows_in_row_tiles"] == 200 + 256 + 512
    assert g1["weight_stream_bytes"] == 3 * (2 * I * d * 2)  # the 100-row expert and two leftovers
    assert g2["rows_in_row_tiles"] == 200 + 256 + 512
    assert g2["weight_stream_bytes"] == 3 * (d * I * 2)      # the 100-row expert and two leftovers
    rate = 2 * 8192 * 1000.0e6
    assert abs(g1["tensor_ms"] - 1e3 * 4.0 * d * I * 968 / rate) < 1e-3
    assert abs(g2["stream_ms"] - 1e3 * 3 * d * I * 2 / 1e9) < 1e-3
    assert g1["frac"] == round(g1["t_bound_ms"] / 1.0, 4)
    # no clock measured for a GEMM: no entry
    assert bench.gemm_phase_roofline(counts, d, I, False, {"gemm1_swiglu": None}, 2, 1.0, {}) == {}


def test_clock_summary_reports_load_clock_reasons_and_power_limit():
    """The `clocks` block: the median SM clock of the samples under load (power above half the
    largest sample), the throttle reasons seen active, and the enforced power limit."""
    sys.path.insert(0, str(ROOT))
    import bench
    rows = [["t", "GPU-x", "1965", "1965", "120.0", "0x0", "Not Active", "Not Active", "Not Active", "Not Active", "1000.00"],
            ["t", "GPU-x", "1300", "1965", "990.0", "0x4", "Not Active", "Not Active", "Not Active", "Active", "1000.00"],
            ["t", "GPU-x", "1400", "1965", "960.0", "0x4", "Not Active", "Not Active", "Not Active", "Active", "1000.00"]]
    c = bench.ClockSampler.summarize(rows)
    assert c["sm_mhz"] == 1350.0 and c["sm_max_mhz"] == 1965.0
    assert c["reasons"] == ["sw_power_cap"] and c["power_limit_w"] == 1000.0
    assert c["samples"] == 3 and c["samples_under_load"] == 2
    # no sampler output: the block says so instead of inventing a clock
    assert bench.ClockSampler.summarize([])["reasons"] == ["nvidia-smi unavailable"]
