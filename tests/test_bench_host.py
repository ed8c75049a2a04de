"""Host logic of bench.py (no GPU): which bf16 peak the roofline fraction is
taken against, and the per-workload figures derived from one timed run."""
import bench
from backward_lstm_fwd_b200 import synth

PEAKS = {"hbm_gbs": 6552.0, "bf16_tflops": 1638.5, "bf16_tflops_sustained": 1368.2}


def test_burst_peak_only_at_max_clock_without_throttle():
    at_max = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
    assert bench.tensor_peak(PEAKS, at_max)[0] == 1638.5
    assert bench.tensor_peak(PEAKS, dict(at_max, reasons=["sw_power_cap"]))[0] == 1368.2
    assert bench.tensor_peak(PEAKS, dict(at_max, sm_mhz=1500.0))[0] == 1368.2
    assert bench.tensor_peak(PEAKS, None)[0] == 1368.2


def test_config_line():
    w = synth.WORKLOADS["lstm_T256_B128_I1024_H1024_bf16"]
    phases = {"fwd_recur": (2 * 1.28, 2), "bwd_recur": (2 * 1.536, 36), "dW": (0.0, 0)}
    c = bench.config_line(w, 2 * 2.5, phases, 2, 1638.5)
    assert abs(c["ms_per_step"] - 2.5) < 1e-12
    assert abs(c["timesteps_per_s"] - w.rows / 2.5e-3) < 1e-6
    assert abs(c["tflops"] - w.flops / 2.5e-3 / 1e12) < 1e-9
    assert abs(c["us_per_recurrent_step"]["fwd"] - 5.0) < 1e-9
    assert abs(c["us_per_recurrent_step"]["bwd"] - 6.0) < 1e-9
    assert "dW" not in c["phases_ms_per_step"]
