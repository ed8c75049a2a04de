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


def test_split_by_size_balances_copy_streams():
    """The end-to-end leg's copies go to two streams per direction, largest
    first onto the lighter stream: every tensor once, loads within the largest
    item of each other."""
    items = [(134, "dx"), (67, "y"), (33, "dW"), (1, "hT"), (1, "cT"), (0.5, "db")]
    lanes = bench.split_by_size(items, 2)
    assert sorted(k for lane in lanes for k in lane) == sorted(k for _, k in items)
    size = dict((k, v) for v, k in items)
    loads = [sum(size[k] for k in lane) for lane in lanes]
    assert abs(loads[0] - loads[1]) <= max(size.values())
    assert bench.split_by_size([(5, "a")], 2) == [["a"]]  # an empty stream is dropped
