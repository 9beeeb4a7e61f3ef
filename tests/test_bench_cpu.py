"""bench.py helpers that need no GPU: the compact summary of the target
figures that closes the JSON line (the part of the line always kept)."""
import json

import bench


def test_target_summary_picks_every_figure():
    r = {"layer_calls": {"grouped_4_calls": {"frac_hbm": 0.3},
                         "separate_7_calls": {"frac_hbm": 0.26}},
         "more_m1": {"70b_gate_m1": {"frac_hbm": 0.36}, "70b_down_m1": {"frac_hbm": 0.31}},
         "batch": {"sweep_m2": {"frac_hbm": 0.27}, "sweep_m4": {"frac_hbm": 0.21},
                   "sweep_m8": {"frac_hbm": 0.2}, "sweep_m16": {"frac_hbm": 0.14},
                   "70b_gate_m8": {"frac_hbm": 0.21}},
         "prefill": {"prefill_gate": {"frac_bf16_burst": 0.67},
                     "prefill_down": {"frac_bf16_burst": 0.72}}}
    nbit = {"any4": {"frac_hbm": 0.66}}
    table = {"matrices": [{"shape": "8b_q", "gpu_ms": 25.0}, {"shape": "8b_down", "gpu_ms": 380.0}]}
    peaks = {"hbm_gbs": 6543.4, "bf16_tflops": 1637.0}
    t = bench.target_summary(r, nbit, table, peaks)
    assert t["m1_8b_layer_grouped"] == 0.3 and t["m1_70b_gate"] == 0.36
    assert t["m8"] == 0.2 and t["m16"] == 0.14 and t["m8_70b_gate"] == 0.21
    assert t["dequant_8b_gate"] == 0.66 and t["prefill_down_burst"] == 0.72
    assert t["quantize_8b_down_ms"] == 380.0
    assert len(json.dumps(t)) < 700  # stays well inside the kept tail of the line


def test_target_summary_tolerates_missing_details():
    t = bench.target_summary({}, {"error": "x"}, None, {"hbm_gbs": 1.0, "bf16_tflops": 1.0})
    assert t["m1_8b_layer_grouped"] is None and t["dequant_8b_gate"] is None
    assert "quantize_8b_down_ms" not in t
