"""The FLOAT16 data type of "SingleLayerLstmGrad" (LSTM_F16: x, W, b, h0, y,
gates, dy, dhT and dG in IEEE binary16, fp32 accumulation and cell state)
against the fp64 oracle, element by element, on every kernel path an fp16
call takes: the fused forward and the TMEM-weight backward (one launch and
chunked, ragged batch groups), the per-step kernels where those plans do not
fit, the bench-size workload on sampled sequences, and fp16 with the other
options.  Tolerance 2.5e-3 per output tensor (the bf16 figure scaled by the
ratio of the unit roundoffs)."""
import pytest

from backward_lstm_fwd_b200 import binding as L
from backward_lstm_fwd_b200 import synth
from tests.parity_util import (OUTS, assert_within, compare, mask_upstream, run_gpu,
                               run_oracle)

pytestmark = pytest.mark.gpu

# (T, B, I, H) -> (forward path, backward path) of lstm_test_last_paths
CASES = {
    (7, 5, 37, 45): (5, 5),        # persistent CUDA-core kernels (H off the 32-unit grid)
    (4, 130, 128, 128): (3, 5),    # fused forward; persistent CUDA-core backward (H < 512)
    (10, 24, 64, 256): (3, 5),
    (12, 48, 64, 512): (3, 3),     # TMEM-weight kernels, one launch each
    (40, 64, 96, 512): (3, 4),     # backward in 2 chunks, two batch streams
    (64, 200, 96, 512): (3, 3),    # ragged batch groups, 4 chunks
    (3, 37, 64, 640): (3, 3),      # odd count of unit slices
}


@pytest.mark.parametrize("shape", sorted(CASES))
def test_fp16(shape, cuda_device):
    T, B, I, H = shape
    w = synth.custom(T, B, I, H, "fp16", seed=T + 3 * B + H)
    inp = synth.make_inputs(w)
    gpu = run_gpu(inp, cuda_device)
    assert L.test_last_paths() == CASES[shape]
    ref = run_oracle(inp)
    assert_within(compare(gpu, ref, "fp16", OUTS + ("gates", "cells")), "fp16", w.name)


def test_fp16_bench_size_sampled(cuda_device):
    """T=256, B=128, I=H=1024 (the benchmark's shape) in fp16, checked on
    sampled sequences; dW and db with the upstream gradient of the sample only."""
    w = synth.custom(256, 128, 1024, 1024, "fp16", seed=3, dhdc=True)
    idx = [0, 77, 127]
    inp = synth.make_inputs(w)
    gpu = run_gpu(inp, cuda_device)
    assert L.test_last_paths() == (3, 4)
    ref = run_oracle(synth.select_sequences(inp, idx))
    errs = compare(gpu, ref, "fp16", ("y", "hT", "cT", "dx", "dh0", "dc0"), idx=idx)
    assert_within(errs, "fp16", w.name + " per-sequence")
    masked = mask_upstream(inp, idx)
    gpu_m = run_gpu(masked, cuda_device)
    ref_m = run_oracle(synth.select_sequences(masked, idx))
    assert_within(compare(gpu_m, ref_m, "fp16", ("dW", "db")), "fp16", w.name + " dW, db")


@pytest.mark.parametrize("shape", [(9, 6, 24, 40), (40, 64, 96, 512)])
def test_fp16_with_options(shape, cuda_device):
    """fp16 with a length mask, the reverse direction and gate_order "ijfo"."""
    T, B, I, H = shape
    w = synth.custom(T, B, I, H, "fp16", seed=7 * T + H)
    inp = synth.make_inputs(w)
    mask = synth.length_mask(T, B, H, synth.random_lengths(T, B, seed=T * 3 + B), "fp16")
    gpu = run_gpu(inp, cuda_device, mask=mask, reverse=True, ijfo=True)
    ref = run_oracle(inp, mask=mask, reverse=True, ijfo=True)
    assert_within(compare(gpu, ref, "fp16", OUTS + ("gates", "cells")), "fp16",
                  w.name + " mask, reverse, ijfo")
