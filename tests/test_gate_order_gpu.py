"""gate_order "ijfo" (the attribute of "SingleLayerLstmGrad": the 4H rows of
W, b, gates and dG are the row blocks i, j (= g), f, o) through lstm_fwd_ex /
lstm_bwd_ex against the fp64 oracle, element by element, on every kernel path
such a call can take; and the forward against the default order with the f
and g blocks of W and b swapped, which must agree bit for bit (each gate's
dot products are the same sums in the same order).  Tolerance as in the other
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
    (64, 200, 96, 512, "bf16"): (3, 3),   # ragged batch groups, 4 chunks
}


def _swap_fg(a, H, axis=0):
    """Exchange row blocks 1 and 2 (of H rows each) along `axis`."""
    idx = np.r_[0:H, 2 * H:3 * H, H:2 * H, 3 * H:4 * H]
    return a.index_select(axis, torch.as_tensor(idx, device=a.device))


@pytest.mark.parametrize("shape", sorted(CASES))
def test_ijfo(shape, cuda_device):
    T, B, I, H, dt = shape
    w = synth.custom(T, B, I, H, dt, seed=3 * T + B + H)
    inp = synth.make_inputs(w)
    gpu = run_gpu(inp, cuda_device, ijfo=True)
    assert L.test_last_paths() == CASES[shape]
    ref = run_oracle(inp, ijfo=True)
    assert_within(compare(gpu, ref, dt, OUTS + ("gates", "cells")), dt, w.name + " ijfo")


@pytest.mark.parametrize("shape", [(9, 6, 24, 40, "fp32"), (12, 48, 64, 512, "bf16"),
                                   (40, 64, 96, 512, "bf16")])
def test_ijfo_forward_is_ifjo_with_blocks_swapped(shape, cuda_device):
    T, B, I, H, dt = shape
    w = synth.custom(T, B, I, H, dt, seed=T + 7 * B)
    inp = {k: (v.to(cuda_device) if v is not None else None)
           for k, v in synth.make_inputs(w).items()}
    a = L.forward(inp["x"], inp["W"], inp["b"], inp["h0"], inp["c0"], gate_order="ijfo")
    path_a = L.test_last_paths()[0]
    b = L.forward(inp["x"], _swap_fg(inp["W"], H), _swap_fg(inp["b"], H), inp["h0"], inp["c0"])
    torch.cuda.synchronize()
    assert L.test_last_paths()[0] == path_a  # the same kernel ran both
    for k in ("y", "hT", "cT", "cells"):
        assert torch.equal(getattr(a, k), getattr(b, k)), k
    assert torch.equal(_swap_fg(a.gates, H, axis=2), b.gates)


@pytest.mark.parametrize("shape", [(9, 6, 24, 40, "fp32"), (40, 64, 96, 512, "bf16")])
def test_ijfo_reverse_with_length_mask(shape, cuda_device):
    T, B, I, H, dt = shape
    w = synth.custom(T, B, I, H, dt, seed=11 * T + H)
    inp = synth.make_inputs(w)
    mask = synth.length_mask(T, B, H, synth.random_lengths(T, B, seed=T + B), dt)
    gpu = run_gpu(inp, cuda_device, mask=mask, reverse=True, ijfo=True)
    ref = run_oracle(inp, mask=mask, reverse=True, ijfo=True)
    assert_within(compare(gpu, ref, dt, OUTS + ("gates", "cells")), dt,
                  w.name + " ijfo, reverse, mask")
