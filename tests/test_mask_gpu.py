"""Variable length (the seq_length mask input of "SingleLayerLstmGrad"): the CUDA
path through lstm_fwd_masked / lstm_bwd_masked against the fp64 oracle, element
by element, on every kernel path a masked call can take -- the fp32 and bf16
per-step kernels, the TMEM-weight cluster kernels in one launch and in
reverse-time chunks with dW / dx beside them -- with per-sequence lengths
(including 0 and T) and element-wise masks.  Tolerance as in the unmasked
parity tests."""
import numpy as np
import pytest
import torch

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
    (64, 200, 96, 512, "bf16"): (3, 3),   # ragged batch groups, backward in 4 chunks
}


@pytest.mark.parametrize("shape", sorted(CASES))
def test_length_mask(shape, cuda_device):
    T, B, I, H, dt = shape
    w = synth.custom(T, B, I, H, dt, seed=T + B + H)
    inp = synth.make_inputs(w)
    mask = synth.length_mask(T, B, H, synth.random_lengths(T, B, seed=H + T), dt)
    gpu = run_gpu(inp, cuda_device, mask=mask)
    assert L.test_last_paths() == CASES[shape]
    ref = run_oracle(inp, mask=mask)
    assert_within(compare(gpu, ref, dt, OUTS + ("cells",)), dt, w.name + " length mask")


@pytest.mark.parametrize("shape", [(9, 6, 24, 40, "fp32"), (12, 48, 64, 512, "bf16"),
                                   (40, 64, 96, 512, "bf16")])
def test_elementwise_mask(shape, cuda_device):
    T, B, I, H, dt = shape
    w = synth.custom(T, B, I, H, dt, seed=3 * T + H)
    inp = synth.make_inputs(w)
    mask = synth.random_mask(T, B, H, dt, seed=T * H)
    gpu = run_gpu(inp, cuda_device, mask=mask)
    ref = run_oracle(inp, mask=mask)
    assert_within(compare(gpu, ref, dt, OUTS + ("cells",)), dt, w.name + " element mask")


@pytest.mark.parametrize("shape", [(9, 6, 24, 40, "fp32"), (40, 64, 96, 512, "bf16")])
def test_all_ones_mask_is_unmasked(shape, cuda_device):
    """A mask of ones gives the unmasked call's results bit for bit."""
    T, B, I, H, dt = shape
    inp = synth.make_inputs(synth.custom(T, B, I, H, dt, seed=11))
    a = run_gpu(inp, cuda_device)
    b = run_gpu(inp, cuda_device, mask=torch.ones(T, B, H, dtype=synth.torch_dtype(dt)))
    for k in OUTS + ("gates", "cells"):
        np.testing.assert_array_equal(a[k], b[k], err_msg=k)


@pytest.mark.parametrize("dt,H", [("fp32", 40), ("bf16", 512)])
def test_all_padding(dt, H, cuda_device):
    """Nothing real: the state passes through (y = h0 at every step, hT = h0,
    cT = c0), no weight or input gradient, dh0 = dhT + sum_t dy_t, dc0 = dcT."""
    T, B, I = 6, 16, 32
    inp = synth.make_inputs(synth.custom(T, B, I, H, dt, seed=13))
    gpu = run_gpu(inp, cuda_device, mask=torch.zeros(T, B, H, dtype=synth.torch_dtype(dt)))
    h0 = inp["h0"].double().numpy()
    for t in range(T):
        np.testing.assert_array_equal(gpu["y"][t], h0)
    np.testing.assert_array_equal(gpu["hT"], h0)
    np.testing.assert_array_equal(gpu["cT"], inp["c0"].double().numpy())
    assert not gpu["dW"].any() and not gpu["db"].any() and not gpu["dx"].any()
    want = inp["dhT"].double().numpy() + inp["dy"].double().numpy().sum(axis=0)
    np.testing.assert_allclose(gpu["dh0"], want, rtol=1e-5, atol=1e-5)
    np.testing.assert_array_equal(gpu["dc0"], inp["dcT"].double().numpy())
