"""lstm_fwd_noalloc: the forward pass for callers that may not allocate device
memory (a plugin inside a host program that owns the device-memory budget, or
a latency-critical loop that cannot afford cudaMalloc's implicit
synchronisation).  It uses the library's static device scratch instead of a
caller workspace.

Its results must match lstm_fwd with a caller workspace, on two calls in a
row (the second call reuses the scratch the first one left behind).  This file
is collected last, so a run that stops at its first failure has already run
every other test; it also passes on its own in a fresh process."""
import numpy as np
import pytest
import torch

from backward_lstm_fwd_b200 import binding as L
from backward_lstm_fwd_b200 import build as lbuild
from backward_lstm_fwd_b200 import synth
from tests.parity_util import TOL, rel_err


def test_noalloc_rejects_problems_beyond_its_scratch():
    lbuild.build()
    L.load()
    big = L.dims(256, 128, 1024, 1024, L.LSTM_BF16)  # needs ~537 MB of Gx
    assert L.fwd_workspace_size(big) > L.NOALLOC_SCRATCH_BYTES
    fake = 0x10000  # never dereferenced: the size check comes first
    rc = L.lstm_fwd_noalloc(big, fake, fake, None, None, None, fake, fake, fake, fake, fake,
                            stream=0, check=False)
    assert rc == L.LSTM_ERR_UNSUPPORTED


def _outputs(st):
    return {k: getattr(st, k).float().cpu().numpy() for k in ("y", "hT", "cT", "gates", "cells")}


@pytest.mark.gpu
@pytest.mark.parametrize("T,B,I,H,dt", [(16, 32, 64, 128, "bf16"), (9, 5, 24, 40, "fp32"),
                                        (12, 64, 256, 256, "bf16"), (4, 128, 64, 512, "bf16")])
def test_noalloc_matches_lstm_fwd_twice(T, B, I, H, dt, cuda_device):
    lbuild.build()
    w = synth.custom(T, B, I, H, dt, seed=T + B + I + H)
    assert L.fwd_workspace_size(L.dims(T, B, I, H, synth.torch_dtype(dt))) <= \
        L.NOALLOC_SCRATCH_BYTES
    inp = {k: v.to(cuda_device) for k, v in synth.make_inputs(w).items()}
    ref = _outputs(L.forward(inp["x"], inp["W"], inp["b"], inp["h0"], inp["c0"]))
    for call in range(2):
        st = L.State(T, B, I, H, synth.torch_dtype(dt), cuda_device)
        L.lstm_fwd_noalloc(st.dims, inp["x"], inp["W"], inp["b"], inp["h0"], inp["c0"], st.y,
                           st.hT, st.cT, st.gates, st.cells)
        torch.cuda.synchronize()
        out = _outputs(st)
        for k in ref:
            e = rel_err(out[k], ref[k])
            assert e <= TOL[dt], (call, k, e)
