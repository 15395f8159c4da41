"""bench.py's JSON line on the CPU: the reference arm (the oracle timed on the
host cores) prints one line with the contract's keys, for the forward
workload and for the scan gradient, and a non-zero rank prints nothing."""
import contextlib
import io
import json

import bench
import pytest


def _run(argv, env=None, monkeypatch=None):
    if env and monkeypatch:
        for k, v in env.items():
            monkeypatch.setenv(k, v)
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        rc = bench.main(argv)
    assert rc == 0
    lines = [ln for ln in buf.getvalue().splitlines() if ln.strip()]
    return [json.loads(ln) for ln in lines]


KEYS = ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
        "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e")


def _check(line, metric):
    for k in KEYS:
        assert k in line, k
    assert line["metric"] == metric
    assert line["impl"] == "reference"
    assert line["value"] > 0 and line["unit"] == "tokens/s"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert "workload" in line["config"]


def test_reference_arm_forward_line():
    out = _run(["--impl", "reference", "--steps", "1", "--warmup", "0", "--seq", "64"])
    assert len(out) == 1
    _check(out[0], bench.METRIC)


def test_reference_arm_scan_backward_line():
    out = _run(["--impl", "reference", "--scan-backward", "--steps", "1", "--warmup", "0"])
    assert len(out) == 1
    _check(out[0], bench.BWD_METRIC)
    assert out[0]["dtype"] == "f64"


def test_reference_arm_other_ranks_print_nothing(monkeypatch):
    out = _run(["--impl", "reference", "--steps", "1", "--warmup", "0", "--seq", "64"],
               env={"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}, monkeypatch=monkeypatch)
    assert out == []


def test_scan_backward_algorithmic_bytes():
    """114,944 B per position at d_inner 4096: 7 fp32 arrays of E channels
    (u, z, dt_raw, dy read; du, dz, ddt_raw written) and B | C read, dB | dC
    written (32 fp32 each)."""
    assert bench.bwd_bytes_per_token(4096) == 4096 * 7 * 4 + 2 * 32 * 4 == 114944


def test_tensor_peak_follows_the_clock_record():
    """A short timed region at full clock with no power cap is measured against
    the burst cuBLAS peak; a power-capped, long or low-clock run against the
    sustained one; the note says which."""
    peaks = {"hbm_gbs": 6500.0, "bf16_tflops": 1650.0, "bf16_tflops_sustained": 1370.0}
    fast = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
    p, note = bench.tensor_peak(peaks, "measured", fast, 40.0)
    assert p == 1650.0 and "burst" in note
    p, note = bench.tensor_peak(peaks, "measured", dict(fast, reasons=["sw_power_cap"]), 40.0)
    assert p == 1370.0 and "power cap" in note
    p, _ = bench.tensor_peak(peaks, "measured", fast, 4000.0)
    assert p == 1370.0
    p, _ = bench.tensor_peak(peaks, "measured", dict(fast, sm_mhz=1400.0), 40.0)
    assert p == 1370.0
    p, _ = bench.tensor_peak(peaks, "measured", None, 40.0)
    assert p == 1370.0


def test_scan_ceilings_arithmetic():
    """The FP32-pipe ceiling of the scan: 75 operations per (token,
    channel) on 148 SMs x 128 lanes per clock; at 1965 MHz and the serving
    shape (32768 tokens x 4096 channels) that is 0.2704 ms."""
    from reverse_selective_ssm_b200 import synthetic as S
    case = S.make_case(2, weights=False, B=8, L=8)      # only the dims and the token count are read
    case.B, case.L, case.lengths = 8, 4096, None
    out = bench.scan_ceilings(case, 0.6436, {"sm_mhz": 1965.0}, "none")
    assert bench.SCAN_FP32_OPS_PER_TOKEN_CHANNEL == 75
    assert out["fp32_pipe"]["ceiling_ms"] == pytest.approx(75 * 32768 * 4096 / (148 * 128 * 1965e6) * 1e3, rel=1e-3)
    assert out["fp32_pipe"]["frac"] == pytest.approx(out["fp32_pipe"]["ceiling_ms"] / 0.6436, rel=1e-3)
    assert "issue" not in out                             # no committed summary for this workload tag


def test_reference_arm_hook_backward_line():
    out = _run(["--impl", "reference", "--hook-backward", "--steps", "1", "--warmup", "0", "--config", "1",
                "--seq", "32"])
    assert len(out) == 1
    _check(out[0], out[0]["metric"])
    assert "hook backward" in out[0]["metric"]


def test_hook_backward_gemm_flops():
    """Three times the forward's projection flops: the recomputed forward and an
    input- and a weight-gradient GEMM per projection (52.69 MFLOP per token
    per layer at d_model 2048, d_inner 4096, dt_rank 128)."""
    from reverse_selective_ssm_b200 import synthetic as S
    case = S.make_case(1, weights=False, L=8)
    per_token = 2 * (2048 * 8192 + 4096 * 160 + 128 * 4096 + 4096 * 2048)
    assert per_token == 52690944
    assert bench.hook_bwd_gemm_flops(case) == 3 * per_token * 8


def test_cpu_baseline_of_a_one_sequence_batch():
    """The forward line's cpu_baseline samples at most the batch's sequences
    (config 1 and config 0 hold one)."""
    from reverse_selective_ssm_b200 import synthetic as S
    case = S.make_case(0)
    assert case.B == 1
    cb = bench.cpu_baseline(case)
    assert cb["kind"] == "oracle" and cb["value"] > 0 and "[0]" in cb["sample"]
