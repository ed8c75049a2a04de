"""lstm_fwd_noalloc: the forward pass for callers that may not allocate device
memory (a plugin inside a host program that owns the device-memory budget, or
a latency-critical loop that cannot afford cudaMalloc's implicit
synchronisation).  It uses the library's static device scratch instead of a
caller workspace.

It runs the same kernels as lstm_fwd with a caller workspace, so its results
must equal lstm_fwd's bit for bit, on two calls in a row (the second call
reuses the scratch the first one left behind, so a stale byte that the kernels
read would show).  A device-side wait that gives up must be reported by
lstm_fwd_noalloc_status.  This file is collected last, so a run that stops at
its first failure has already run every other test; it also passes on its own
in a fresh process."""
import numpy as np
import pytest
import torch

from backward_lstm_fwd_b200 import binding as L
from backward_lstm_fwd_b200 import build as lbuild
from backward_lstm_fwd_b200 import synth


def test_noalloc_rejects_problems_beyond_its_scratch():
    """An fp32 problem always reads its input projection from the workspace:
    T*B*4H floats of Gx (537 MB here) cannot fit the 32 MiB scratch on any
    device, so the call is refused before any pointer is read."""
    lbuild.build()
    L.load()
    big = L.dims(256, 128, 1024, 1024, L.LSTM_F32)
    assert L.fwd_workspace_size(big) > L.NOALLOC_SCRATCH_BYTES
    fake = 0x10000  # never dereferenced: the size check comes first
    rc = L.lstm_fwd_noalloc(big, fake, fake, None, None, None, fake, fake, fake, fake, fake,
                            stream=0, check=False)
    assert rc == L.LSTM_ERR_UNSUPPORTED


def _outputs(st):
    return {k: getattr(st, k).float().cpu().numpy() for k in ("y", "hT", "cT", "gates", "cells")}


@pytest.mark.gpu
@pytest.mark.parametrize("T,B,I,H,dt", [(16, 32, 64, 128, "bf16"), (9, 5, 24, 40, "fp32"),
                                        (12, 64, 256, 256, "bf16"), (4, 128, 64, 512, "bf16"),
                                        (256, 128, 1024, 1024, "bf16")])
def test_noalloc_matches_lstm_fwd_twice(T, B, I, H, dt, cuda_device):
    """The last shape is the bench workload: on a device where the fused
    forward kernel runs, it needs only the control block of the scratch."""
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
        assert L.lstm_fwd_noalloc_status() == L.LSTM_OK
        out = _outputs(st)
        for k in ref:
            np.testing.assert_array_equal(out[k], ref[k], err_msg=f"call {call}, {k}")


@pytest.mark.gpu
def test_noalloc_status_reports_a_wait_that_gave_up(cuda_device):
    """A persistent kernel whose CTA 0 never signals its step barrier gives up
    after its bounded wait; lstm_fwd_noalloc_status reports LSTM_ERR_TIMEOUT
    once (reading clears it), and the next call runs normally."""
    lbuild.build()
    T, B, I, H = 6, 128, 64, 128
    w = synth.custom(T, B, I, H, "bf16", seed=13)
    inp = {k: v.to(cuda_device) for k, v in synth.make_inputs(w).items()}
    ref = _outputs(L.forward(inp["x"], inp["W"], inp["b"], inp["h0"], inp["c0"]))
    st = L.State(T, B, I, H, torch.bfloat16, cuda_device)
    try:
        L.test_set_wait_fault(0, 50_000_000)  # waits give up after 50 ms
        L.lstm_fwd_noalloc(st.dims, inp["x"], inp["W"], inp["b"], inp["h0"], inp["c0"], st.y,
                           st.hT, st.cT, st.gates, st.cells)
        assert L.lstm_fwd_noalloc_status() == L.LSTM_ERR_TIMEOUT
        assert L.lstm_fwd_noalloc_status() == L.LSTM_OK
    finally:
        L.test_set_wait_fault(-1, 0)
    L.lstm_fwd_noalloc(st.dims, inp["x"], inp["W"], inp["b"], inp["h0"], inp["c0"], st.y,
                       st.hT, st.cT, st.gates, st.cells)
    assert L.lstm_fwd_noalloc_status() == L.LSTM_OK
    out = _outputs(st)
    for k in ref:
        np.testing.assert_array_equal(out[k], ref[k], err_msg=k)
