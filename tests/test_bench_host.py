"""CPU: host logic of bench.py -- the reference arm's JSON line (with the oracle
sample stubbed, so that the contract is checked in milliseconds), the parsing
of the nvidia-smi clock record, and the peak figures' fallback."""
import json
import types

import pytest

import bench
from bit_fp8_attention_prep_b200 import synth


def _args(**kw):
    base = dict(gpus=1, steps=3, warmup=3, impl="reference", workload="minimax_h56", k_p=8, no_extras=False,
                extras="all", head_chunk=4, sweep=None)
    base.update(kw)
    return types.SimpleNamespace(**base)


def test_reference_line_has_the_contract_keys(monkeypatch, capsys):
    calls = []

    def fake_sample(cfg, S_sample, rows, seed=0):
        calls.append(S_sample)
        return 20.0, 0.5, f"stub over {S_sample} tokens"

    monkeypatch.setattr(bench, "oracle_sample", fake_sample)
    monkeypatch.setattr(bench, "oracle_cores", lambda: 1)
    monkeypatch.delenv("RANK", raising=False)
    cfg = synth.workload("minimax_h56")
    bench.run_reference(_args(), cfg)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert len(calls) == 6                                   # warm-up and timed steps
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC and line["unit"] == bench.UNIT
    assert line["ms_per_step"] == pytest.approx(20.0e3)
    assert line["value"] == pytest.approx(bench.flops_of(cfg) / 20.0 / 1e12)
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["cpu_baseline"]["cores"] == 1
    assert line["e2e"] == {"value": line["value"], "unit": bench.UNIT, "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert line["config"]["workload"] == "minimax_h56" and line["config"]["S"] == 73397


def test_reference_arm_prints_nothing_off_rank_zero(monkeypatch, capsys):
    monkeypatch.setattr(bench, "oracle_sample", lambda *a, **k: pytest.fail("rank 1 must not run the oracle"))
    monkeypatch.setenv("RANK", "1")
    bench.run_reference(_args(), synth.workload("minimax_h56"))
    assert capsys.readouterr().out == ""


def test_clock_record_parsing():
    out = "\n".join([
        "1650, 1965, 900.1, Not Active, Not Active, Not Active, Active",
        "1700, 1965, 950.0, Not Active, Not Active, Not Active, Active",
        "1680, 1965, 930.0, Not Active, Active, Not Active, Not Active",
        "garbage line",
        "[N/A], 1965, 1.0, Not Active, Not Active, Not Active, Not Active",
    ])

    class FakeProc:
        def terminate(self):
            pass

        def communicate(self, timeout=None):
            return out, ""

    cs = bench.ClockSampler(0)
    cs.proc = FakeProc()
    rec = cs.stop()
    assert rec == {"sm_mhz": 1680.0, "sm_max_mhz": 1965.0, "reasons": ["hw_thermal_slowdown", "sw_power_cap"],
                   "samples": 3}
    assert bench.ClockSampler(0).stop() is None            # never started


def test_peaks_fallback(monkeypatch, tmp_path):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    p = bench.load_peaks()
    assert p["source"] == "fallback" and p["hbm"] == bench.FALLBACK_HBM_GBS
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps(
        {"hbm_gbs": 6000.0, "bf16_tflops": 1500.0, "bf16_tflops_sustained": 1300.0}))
    p = bench.load_peaks()
    assert p == dict(bf16_sustained=1300.0, bf16_burst=1500.0, hbm=6000.0, source="measured")


def test_oracle_on_several_cores_shares_the_slices(monkeypatch):
    # two spawned processes, each timing a tiny oracle sample: the workload estimate
    # is the mean per-process estimate over the process count
    monkeypatch.setattr(bench, "oracle_cores", lambda: 2)
    cfg = synth.workload("tiny")
    full, took, desc, cores = bench.oracle_sample_cores(cfg, 256, 8)
    assert cores == 2 and full > 0 and took > 0 and "2 processes" in desc
