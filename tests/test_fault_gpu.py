"""Failure detection without a GPU fault: a persistent recurrent kernel whose
CTA 0 never signals its step barrier must give up after its bounded wait,
record LSTM_ERR_TIMEOUT in the workspace status word (read by lstm_status), and
leave the context usable -- the next normal call succeeds and matches the
oracle."""
import pytest
import torch

from backward_lstm_fwd_b200 import binding as L
from backward_lstm_fwd_b200 import build as lbuild
from backward_lstm_fwd_b200 import synth
from tests.parity_util import assert_within, compare, run_gpu, run_oracle

pytestmark = pytest.mark.gpu


def test_missing_arrival_times_out_and_recovers(cuda_device):
    lbuild.build()
    w = synth.custom(6, 32, 64, 64, "bf16", seed=11)
    inp = {k: v.to(cuda_device) for k, v in synth.make_inputs(w).items()}
    T, B, I, H = w.T, w.B, w.I, w.H
    st = L.State(T, B, I, H, torch.bfloat16, cuda_device)
    ws = L.empty_workspace(L.fwd_workspace_size(st.dims), cuda_device)
    try:
        L.test_set_wait_fault(0, 50_000_000)  # 50 ms
        L.lstm_fwd(st.dims, inp["x"], inp["W"], inp["b"], inp["h0"], inp["c0"], st.y, st.hT,
                   st.cT, st.gates, st.cells, ws)
        assert L.lstm_status(ws) == L.LSTM_ERR_TIMEOUT
        assert L.lstm_status(ws) == L.LSTM_OK  # reading clears the word
    finally:
        L.test_set_wait_fault(-1, 0)
    # the context is still usable and the next call is correct
    out = run_gpu(synth.make_inputs(w), cuda_device)
    assert_within(compare(out, run_oracle(synth.make_inputs(w)), "bf16"), "bf16", "after fault")
