"""The benchmark's work model and roofline arithmetic (no GPU): the counts
behind every TFLOP/s and % of roofline that bench.py reports."""
import argparse
import math
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from ispa_synth import C1, C2, C3  # noqa: E402


def test_chunk_step_work_matches_the_stated_counts():
    """1.3B chunk: attention 4 Nq Nk d over sink + local + history keys (the
    number the attention roofline divides by), Gram 4 N d^2, solve
    (1/3 + 4) d^3; the error pass (a reduction over resident matrices, W W^T
    formed once at load) is credited with no flops."""
    w = bench.step_work(C1)
    nq, nk, d = 4680, 1560 + 4680 + 14040, 1536
    assert w["attention"] == 4.0 * nq * nk * d == 583129497600.0
    assert w["gram"] == 4.0 * 4680 * d * d
    assert math.isclose(w["solve"], (1.0 / 3.0 + 4.0) * d ** 3)
    assert w["error"] == 0.0


def test_warmup_step_work_sums_every_chunk_and_layer():
    """1.3B warmup: four chunks with 0, 3, 6, 9 frames of history, 30 layers;
    the Gram counts every warmup row once (4 x 4680 = 18720)."""
    w = bench.step_work(C2)
    d, tpf = 1536, 1560
    attn = sum(4.0 * 4680 * (1560 + 4680 + 3 * c * tpf) * d for c in range(4))
    assert w["attention"] == pytest.approx(attn * 30)
    assert w["gram"] == pytest.approx(4.0 * 18720 * d * d * 30)
    assert w["solve"] == pytest.approx((1.0 / 3.0 + 4.0) * d ** 3 * 30)


def test_absorb_roofline_is_the_sum_of_its_parts():
    """T* per layer = Gram at the tf32 rate + solve at a third of it + error
    reads at the HBM rate; frac = T* / measured."""
    tf32, _ = bench.tf32_peak(1600.0)
    d, n = C3.d, C3.warmup_rows
    r = bench.absorb_roofline(C3, gram_ms=40 * 3.5, solve_ms=40 * 5.0, bf16_peak=1600.0,
                              hbm_peak=6500.0)
    t_gram = 4.0 * n * d * d / (tf32 * 1e12) * 1e3
    t_solve = (1.0 / 3.0 + 4.0) * d ** 3 / (tf32 / 3.0 * 1e12) * 1e3
    t_err = 6.0 * d * d * 4 / (6500.0 * 1e9) * 1e3
    assert r["t_star_ms_per_layer"] == pytest.approx(t_gram + t_solve + t_err, abs=1e-4)
    assert r["achieved_ms_per_layer"] == pytest.approx(8.5)
    assert r["frac"] == pytest.approx((t_gram + t_solve + t_err) / 8.5, abs=1e-4)
    # context: the same flops all at the bf16 rate, the error reads unchanged
    t_bf16 = (4.0 * n * d * d + (1.0 / 3.0 + 4.0) * d ** 3) / (1600.0 * 1e12) * 1e3 + t_err
    assert r["bf16_only"]["t_ms_per_layer"] == pytest.approx(t_bf16, abs=1e-4)
    assert r["bf16_only"]["frac"] == pytest.approx(t_bf16 / 8.5, abs=1e-4)
    assert r["bf16_only"]["t_ms_per_layer"] < r["t_star_ms_per_layer"]


@pytest.mark.parametrize("config,layers,k", [("c2", 4, 2), ("c3", 2, 1), ("c2", 30, 15)])
def test_layer_override_keeps_the_fraction_of_l_layers(config, layers, k):
    args = argparse.Namespace(config=config, layers=layers)
    cfg = bench.workload(args)
    assert cfg.layers == layers and cfg.select_k == k


def test_attention_algorithmic_bytes():
    """Bytes the attention must move per layer: Q, K, V in (bf16), A_loc and
    D out (fp32), A_full out (bf16), three LSE rows per head (fp32). The 1.3B
    chunk: 14.4 + 124.6 + 71.9 + 0.7 = 211.6 MB."""
    assert bench.attention_bytes(C1) == pytest.approx(211.6e6, rel=1e-3)
    d = 1536
    per_chunk = [(4680 + 2 * (1560 + 4680 + 3 * c * 1560)) * d * 2 + 4680 * d * 10 + 3 * 12 * 4680 * 4
                 for c in range(4)]
    assert bench.attention_bytes(C2) == pytest.approx(sum(per_chunk))


def test_bench_line_config_is_shared_by_both_arms():
    """The reference arm prints the same ``config`` object as ours."""
    a = bench.config_of(C2, 1, False, 15)
    assert a["workload"] == C2.name and a["layers"] == 30 and a["history"] == [0, 4680, 9360, 14040]
    assert a["parallelism"] == "single GPU"


def test_clock_record_rejection():
    """A timed region is measured again when its clock record shows a slowdown
    other than the power cap, or SM clocks far below their maximum with no
    reason active (a clock lock left behind); the power cap alone is kept."""
    rec = lambda mhz, reasons: {"sm_mhz": mhz, "sm_max_mhz": 1965.0, "reasons": reasons}
    assert not bench.clocks_rejected(None)
    assert not bench.clocks_rejected(rec(1700.0, ["sw_power_cap"]))
    assert not bench.clocks_rejected(rec(1900.0, []))
    assert bench.clocks_rejected(rec(1900.0, ["hw_slowdown"]))
    assert bench.clocks_rejected(rec(1500.0, ["sw_power_cap", "sw_thermal_slowdown"]))
    assert bench.clocks_rejected(rec(1000.0, []))
    assert not bench.clocks_rejected(rec(1000.0, ["sw_power_cap"]))
    assert bench.any_over_ranks(True, 1) and not bench.any_over_ranks(False, 1)


def test_oracle_baseline_reports_its_stages_and_threads():
    """The CPU baseline's per-stage extrapolated seconds add up to its full
    step, and it states the host cores and BLAS threads it ran with."""
    from ispa_synth import CONFIGS
    r = bench.oracle_throughput(CONFIGS["c0"], budget_s=0.0)
    st = r["stage_seconds_per_full_step"]
    assert set(st) == {"attention", "gram", "solve"}        # the error stage is credited no flops
    assert sum(st.values()) == pytest.approx(r["seconds_per_full_step"], abs=5e-3)
    assert r["host_cores"] >= 1 and r["cores"] >= 1
    assert r["kind"] == "oracle" and r["value"] > 0


def test_error_pass_bytes():
    """The batched error pass reads G and S on and above the tile diagonal and
    R, W W^T, Delta W and B in full, fp32: about 5 d^2 floats a layer (an ncu
    capture of the pass over four d = 1536 layers read 191.9 MB)."""
    for cfg in (C1, C3):
        d, t = cfg.d, cfg.d // 128
        tiles_upper = t * (t + 1) // 2
        assert bench.error_bytes(cfg) == 4 * (2 * tiles_upper * 128 ** 2 + 4 * d * d)
    assert bench.error_bytes(C1) == pytest.approx(47.97e6, rel=1e-3)     # d = 1536
    assert bench.error_bytes(C3) == pytest.approx(526.9e6, rel=1e-3)     # d = 5120
