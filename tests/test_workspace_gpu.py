"""The forward's plan-aware workspace size on a B200: the fused forward kernel
needs only the 256-byte control block, and a call that is forced onto a plan
with the fp32 input projection (LSTM_FWD_FUSED_X=0) either gets the larger
workspace and matches the oracle, or is refused with LSTM_ERR_WORKSPACE."""
import pytest
import torch

from backward_lstm_fwd_b200 import binding as L
from backward_lstm_fwd_b200 import build as lbuild
from backward_lstm_fwd_b200 import synth
from tests.parity_util import assert_within, compare, run_gpu, run_oracle

pytestmark = pytest.mark.gpu


def test_fused_plan_needs_the_control_block_only(cuda_device):
    lbuild.build()
    d = L.dims(256, 128, 1024, 1024, L.LSTM_BF16)
    assert L.fwd_workspace_size(d) == 256
    assert L.fwd_workspace_size(d, mask=torch.empty(1)) == 256
    assert L.fwd_workspace_size_max(d) >= 256 * 128 * 4096 * 4
    # fp32 always reads Gx from the workspace
    f = L.dims(256, 128, 1024, 1024, L.LSTM_F32)
    assert L.fwd_workspace_size(f) == L.fwd_workspace_size_max(f)


@pytest.mark.parametrize("T,B,I,H", [(6, 128, 64, 128), (5, 40, 96, 512)])
def test_forced_gx_plan(T, B, I, H, cuda_device, monkeypatch):
    lbuild.build()
    w = synth.custom(T, B, I, H, "bf16", seed=T + B + H)
    inp = synth.make_inputs(w)
    dev = {k: v.to(cuda_device) for k, v in inp.items()}
    st = L.State(T, B, I, H, torch.bfloat16, cuda_device)
    small = L.empty_workspace(L.fwd_workspace_size(st.dims), cuda_device)
    assert small.numel() == 256
    # the fused plan runs in the small workspace
    L.lstm_fwd(st.dims, dev["x"], dev["W"], dev["b"], dev["h0"], dev["c0"], st.y, st.hT, st.cT,
               st.gates, st.cells, small)
    assert L.test_last_paths()[0] == 3
    monkeypatch.setenv("LSTM_FWD_FUSED_X", "0")
    assert L.fwd_workspace_size(st.dims) == L.fwd_workspace_size_max(st.dims) > 256
    rc = L.lstm_fwd(st.dims, dev["x"], dev["W"], dev["b"], dev["h0"], dev["c0"], st.y, st.hT,
                    st.cT, st.gates, st.cells, small, check=False)
    assert rc == L.LSTM_ERR_WORKSPACE
    out = run_gpu(inp, cuda_device)  # sizes its workspace by the query: the Gx plan
    assert L.test_last_paths()[0] != 3
    assert_within(compare(out, run_oracle(inp), "bf16"), "bf16", "Gx plan")
