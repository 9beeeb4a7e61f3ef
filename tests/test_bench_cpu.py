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


class _FakeProc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        pass


def test_clock_sampler_reads_sm_and_memory_clocks(tmp_path):
    import os
    c = bench.ClockSampler(0)
    c.path = str(tmp_path / "clocks.csv")
    with open(c.path, "w") as f:
        f.write("0, 1965, 1965, 512.0, 0x0, Not Active, Not Active, Not Active, Not Active, 3996\n")
        f.write("0, 1800, 1965, 990.5, 0x4, Not Active, Not Active, Not Active, Active, 3996\n")
        f.write("0, 1965, 1965, 700.0, 0x0, Not Active, Not Active, Not Active, Not Active, 3996\n")
        f.write("garbage line\n")
    c.proc = _FakeProc()
    c.fh = open(os.devnull, "w")
    got = c.stop()
    assert got == {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"],
                   "samples": 3, "mem_mhz": 3996.0}
    assert not os.path.exists(c.path)


def test_oracle_single_thread_restores_the_thread_count():
    import oracle
    before = oracle.num_threads()
    got = bench.oracle_single_thread()
    assert oracle.num_threads() == before
    assert got["cores"] == 1 and set(got["configs"]) == {"tiny", "8b_gate"}
    for v in got["configs"].values():
        assert v["dequant_s"] > 0 and v["matmul_s"] > 0 and v["GB/s"] > 0
