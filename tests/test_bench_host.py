"""Host-side arithmetic of bench.py, on CPU: the rates reported for a timed
shape (tokens/s, TFLOP/s in the FA convention and in the strict count, the
per-pass rates) and the choice of peak (measured file, else the fallback)."""
import json

import pytest

import bench
from mixed_head_causal_b200 import inputs as I


def test_rates_of_a_fwd_bwd_shape():
    w = I.WORKLOADS["124m_b8_t4096_r25"]
    t = {"fwd_ms": 0.25, "bwd_ms": 0.5, "step_ms": 0.75}
    res = bench.rates(w, t, {"bf16_tflops": 1000.0})
    unit = 8 * 64 * 4096 ** 2  # B d T^2
    assert res["tokens_per_s"] == pytest.approx(8 * 4096 / 0.75e-3)
    # 9 ordinary heads at 7 units (2 fwd + 5 bwd), 3 replaced at 2
    assert res["tflops"] == pytest.approx(unit * (9 * 7 + 3 * 2) / 0.75e-3 / 1e12)
    assert res["frac_of_peak"] == pytest.approx(res["tflops"] / 1000.0)
    assert res["fwd_tflops"] == pytest.approx(unit * (9 * 2 + 3) / 0.25e-3 / 1e12)
    assert res["bwd_tflops"] == pytest.approx(unit * (9 * 5 + 3) / 0.5e-3 / 1e12)
    # the strict count drops the backward's recompute of Q K^T: 6 units per ordinary head
    assert res["tflops_strict"] / res["tflops"] == pytest.approx((9 * 6 + 3 * 2) / (9 * 7 + 3 * 2))


def test_rates_of_a_forward_only_shape():
    w = I.WORKLOADS["prefill_124m_b64_t4096"]
    res = bench.rates(w, {"fwd_ms": 2.0, "step_ms": 2.0}, {"bf16_tflops": 1590.0})
    assert "bwd_tflops" not in res and "tflops_strict" not in res
    assert res["tflops"] == pytest.approx(64 * 64 * 4096 ** 2 * (9 * 2 + 3) / 2.0e-3 / 1e12)
    assert res["passes"] == "fwd"


def test_peak_is_the_measured_file_else_the_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    pk = bench.peaks()
    assert pk["src"] == "fallback" and pk["bf16_tflops"] == 1590.0 and pk["hbm_gbs"] == 6650.0
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 7000.0, "bf16_tflops": 1615.5}))
    pk = bench.peaks()
    assert pk["src"] == "measured" and pk["bf16_tflops"] == 1615.5
    assert pk["bf16_tflops_sustained"] == 1615.5  # no sustained figure: the burst one stands in
