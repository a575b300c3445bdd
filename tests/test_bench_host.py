"""bench.py's host-side parts, on the CPU: the algorithmic FLOP and byte
counts the roofline divides by, the peak file with its fallback, the summary
of the clock samples taken during the timed region, and the reference arm
(the CPU oracle timed on a row sample) with its JSON line."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_prefill_flops_is_one_causal_pass():
    # 4 * B * Hq * D * L(L+1)/2: QK^T and PV over the causal triangle
    assert bench.prefill_flops(1, 32, 128, 131072) == 4 * 32 * 128 * 131072 * 131073 / 2
    assert abs(bench.prefill_flops(1, 32, 128, 131072) - 1.407e14) / 1.407e14 < 1e-3
    assert bench.prefill_flops(2, 1, 64, 1) == 2 * 4 * 64
    # the sampled-row count agrees with the closed form when every row is taken
    L, D = 50, 16
    assert bench.rows_flops(D, range(L)) == bench.prefill_flops(1, 1, D, L)


def test_kv_bytes_is_k_and_v_in_bf16():
    assert bench.kv_bytes(1, 8, 128, 131072) == 536870912
    assert bench.kv_bytes(3, 2, 64, 10) == 3 * 10 * 2 * 64 * 2 * 2


def test_peaks_fall_back_without_the_measured_file(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    hbm, bf16, sustained, kind = bench.peaks()
    assert kind == "fallback" and (hbm, bf16, sustained) == (6650.0, 1590.0, 1400.0)
    (tmp_path / "MEASURED_PEAKS.json").write_text(
        json.dumps({"hbm_gbs": 6500.5, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1390.0}))
    assert bench.peaks() == (6500.5, 1600.0, 1390.0, "measured")
    (tmp_path / "MEASURED_PEAKS.json").write_text(
        json.dumps({"hbm_gbs": 6500.5, "bf16_tflops": 1600.0}))
    assert bench.peaks() == (6500.5, 1600.0, 1600.0, "measured")


def test_clock_samples_summary():
    lines = [
        "0, 1800, 1965, 900.1, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n",
        "0, 1600, 1965, 990.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n",
        "garbage line\n",
        "0, [N/A], 1965, 990.0, 0x0, Not Active, Not Active, Not Active, Not Active\n",
        "0, 1700, 1965, 950.0, 0x0, Not Active, Active, Not Active, Not Active\n",
    ]
    got = bench.parse_clock_samples(lines)
    assert got == {"sm_mhz": 1700.0, "sm_max_mhz": 1965.0,
                   "reasons": ["hw_thermal_slowdown", "sw_power_cap"], "samples": 3}
    assert bench.parse_clock_samples(["", "x, y\n"]) is None


def test_single_rank_helpers_need_no_process_group():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.rank_seed(7, 0) != bench.rank_seed(7, 1)


def _bench(env_extra, *argv):
    import subprocess
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *argv],
                          capture_output=True, text=True, env=env, timeout=600)


def test_reference_arm_prints_the_contract_line():
    """`bench.py --impl reference` times the CPU oracle on a bounded row
    sample and prints one JSON line with the base contract's keys."""
    res = _bench({}, "--impl", "reference", "--steps", "1", "--warmup", "3")
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["metric"] == bench.METRIC
    assert rec["value"] > 0 and rec["unit"] == "TFLOP/s" and rec["higher_is_better"] is True
    assert (rec["steps"], rec["warmup"], rec["n_gpus"]) == (1, 3, 1)
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["cpu_baseline"]["cores"] >= 1
    assert rec["cpu_baseline"]["value"] == rec["value"]
    assert rec["e2e"] == {"value": rec["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                          "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_exit_quietly():
    res = _bench({"RANK": "1", "WORLD_SIZE": "2"}, "--impl", "reference", "--steps", "1",
                 "--warmup", "3")
    assert res.returncode == 0, res.stderr[-2000:]
    assert not [l for l in res.stdout.splitlines() if l.startswith("{")]
