"""Failure detection without a GPU fault: a persistent recurrent kernel whose
CTA 0 never signals its step barrier must give up after its bounded wait,
record LSTM_ERR_TIMEOUT in the workspace status word (read by lstm_status), and
leave the context usable -- the next normal call succeeds and matches the
oracle.  Covered for the K-resident kernels (H = 64), the cluster kernels
(H = 256: forward clusters of 4, backward clusters of 8), the backward
cluster kernel with the weights in tensor memory with two decoupled batch
streams per group (H = 512, 1024) and with one (forced), and the fused
forward with one and with two batch streams per cluster."""
import pytest
import torch

from backward_lstm_fwd_b200 import binding as L
from backward_lstm_fwd_b200 import build as lbuild
from backward_lstm_fwd_b200 import synth
from tests.parity_util import assert_within, compare, run_gpu, run_oracle

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("H,T,B,streams", [(64, 6, 32, 2), (256, 6, 32, 2), (512, 6, 32, 2),
                                           (512, 40, 32, 2), (512, 6, 128, 2), (1024, 6, 128, 2),
                                           (1024, 40, 128, 1)])
def test_missing_arrival_times_out_and_recovers(H, T, B, streams, cuda_device, monkeypatch):
    """T = 40 runs the backward in reverse-time chunks with dW / dx beside them;
    B = 128 runs the forward with two interleaved batch streams per cluster (at
    H = 1024 with the bench workload's cluster grid)."""
    lbuild.build()
    if streams == 1:
        monkeypatch.setenv("LSTM_BWD_STREAMS", "1")
    w = synth.custom(T, B, 64, H, "bf16", seed=11)
    inp = {k: v.to(cuda_device) for k, v in synth.make_inputs(w).items()}
    I = w.I
    st = L.State(T, B, I, H, torch.bfloat16, cuda_device)
    gr = L.Grads(T, B, I, H, cuda_device)
    wsf = L.empty_workspace(L.fwd_workspace_size(st.dims), cuda_device)
    wsb = L.empty_workspace(L.bwd_workspace_size(st.dims), cuda_device)
    try:
        L.test_set_wait_fault(0, 50_000_000)  # CTA 0 never arrives; waits give up after 50 ms
        L.lstm_fwd(st.dims, inp["x"], inp["W"], inp["b"], inp["h0"], inp["c0"], st.y, st.hT,
                   st.cT, st.gates, st.cells, wsf)
        assert L.lstm_status(wsf) == L.LSTM_ERR_TIMEOUT
        assert L.lstm_status(wsf) == L.LSTM_OK  # reading clears the word
        L.lstm_bwd(st.dims, inp["dy"], inp["dhT"], inp["dcT"], inp["x"], inp["W"], inp["h0"],
                   inp["c0"], st.y, st.gates, st.cells, gr.dx, gr.dW, gr.db, gr.dh0, gr.dc0, wsb)
        assert L.lstm_status(wsb) == L.LSTM_ERR_TIMEOUT
        assert L.test_last_paths()[1] == {64: 1, 256: 2, 512: 4, 1024: 4 if streams == 2 else 3}[H]
    finally:
        L.test_set_wait_fault(-1, 0)
    # the context is still usable and the next call is correct
    out = run_gpu(synth.make_inputs(w), cuda_device)
    assert_within(compare(out, run_oracle(synth.make_inputs(w)), "bf16"), "bf16", "after fault")


@pytest.mark.parametrize("dt,H", [("fp32", 256), ("bf16", 45)])
def test_persistent_cuda_core_time_out_and_recover(dt, H, cuda_device):
    """The persistent CUDA-core recurrences (fp32, and 16-bit shapes off the
    tensor-core grids) meet at a grid-wide step counter: with CTA 0 never
    arriving, both give up, report LSTM_ERR_TIMEOUT, and the next call runs
    (fp32 at H = 256 with the K axis split over clusters, bf16 at H = 45 without)."""
    lbuild.build()
    T, B, I = 6, 32, 37
    w = synth.custom(T, B, I, H, dt, seed=13)
    inp = {k: v.to(cuda_device) for k, v in synth.make_inputs(w).items()}
    cd = synth.torch_dtype(dt)
    st = L.State(T, B, I, H, cd, cuda_device)
    gr = L.Grads(T, B, I, H, cuda_device)
    wsf = L.empty_workspace(L.fwd_workspace_size(st.dims), cuda_device)
    wsb = L.empty_workspace(L.bwd_workspace_size(st.dims), cuda_device)
    try:
        L.test_set_wait_fault(0, 50_000_000)
        L.lstm_fwd(st.dims, inp["x"], inp["W"], inp["b"], inp["h0"], inp["c0"], st.y, st.hT,
                   st.cT, st.gates, st.cells, wsf)
        assert L.lstm_status(wsf) == L.LSTM_ERR_TIMEOUT
        L.lstm_bwd(st.dims, inp["dy"], inp["dhT"], inp["dcT"], inp["x"], inp["W"], inp["h0"],
                   inp["c0"], st.y, st.gates, st.cells, gr.dx, gr.dW, gr.db, gr.dh0, gr.dc0, wsb)
        assert L.lstm_status(wsb) == L.LSTM_ERR_TIMEOUT
        assert L.test_last_paths() == (5, 5)
        if dt == "fp32":
            # K split over clusters in both directions: the time-out also
            # exercises the exit path in which every CTA of a cluster waits for
            # its peers before leaving
            assert min(L.test_last_persist_split()) > 1
    finally:
        L.test_set_wait_fault(-1, 0)
    out = run_gpu(synth.make_inputs(w), cuda_device)
    assert_within(compare(out, run_oracle(synth.make_inputs(w)), dt), dt, "after fault")
