"""Reverse direction (the "direction" attribute of "SingleLayerLstmGrad",
"REDIRECTIONAL": the recurrence runs over t = T-1 .. 0) through lstm_fwd_ex /
lstm_bwd_ex against the fp64 oracle, element by element, on every kernel path
a reverse-direction call can take, alone and with a variable-length mask.
Tolerance as in the other parity tests."""
import pytest

from backward_lstm_fwd_b200 import binding as L
from backward_lstm_fwd_b200 import synth
from tests.parity_util import OUTS, assert_within, compare, run_gpu, run_oracle

pytestmark = pytest.mark.gpu

# (T, B, I, H, dtype) -> (forward path, backward path) of lstm_test_last_paths
CASES = {
    (9, 6, 24, 40, "fp32"): (5, 5),       # persistent CUDA-core kernels, fp32
    (7, 5, 37, 45, "bf16"): (5, 5),       # persistent CUDA-core kernels, bf16 off the tensor-core grid
    (10, 24, 64, 256, "bf16"): (3, 5),    # fused forward; persistent CUDA-core backward
    (12, 48, 64, 512, "bf16"): (3, 3),    # TMEM-weight kernels, one launch each
    (40, 64, 96, 512, "bf16"): (3, 4),    # backward in 2 chunks, two batch streams
    (64, 200, 96, 512, "bf16"): (3, 3),   # ragged batch groups, 4 chunks
}


@pytest.mark.parametrize("shape", sorted(CASES))
def test_reverse(shape, cuda_device):
    T, B, I, H, dt = shape
    w = synth.custom(T, B, I, H, dt, seed=2 * T + B + H)
    inp = synth.make_inputs(w)
    gpu = run_gpu(inp, cuda_device, reverse=True)
    assert L.test_last_paths() == CASES[shape]
    ref = run_oracle(inp, reverse=True)
    assert_within(compare(gpu, ref, dt, OUTS + ("gates", "cells")), dt, w.name + " reverse")


@pytest.mark.parametrize("shape", [(9, 6, 24, 40, "fp32"), (40, 64, 96, 512, "bf16")])
def test_reverse_with_length_mask(shape, cuda_device):
    T, B, I, H, dt = shape
    w = synth.custom(T, B, I, H, dt, seed=5 * T + H)
    inp = synth.make_inputs(w)
    mask = synth.length_mask(T, B, H, synth.random_lengths(T, B, seed=T * B), dt)
    gpu = run_gpu(inp, cuda_device, mask=mask, reverse=True)
    ref = run_oracle(inp, mask=mask, reverse=True)
    assert_within(compare(gpu, ref, dt, OUTS + ("cells",)), dt, w.name + " reverse, mask")
