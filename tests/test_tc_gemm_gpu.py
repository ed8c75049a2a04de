"""The tcgen05 / TMA GEMM core in isolation (through the test hook of
include/liblstm_testing.h) against torch.matmul on the same bf16 operands,
for every operand majorness the LSTM path uses, with ragged M, N and K."""
import pytest
import torch

from backward_lstm_fwd_b200 import binding as L
from backward_lstm_fwd_b200 import build as lbuild

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("a_mn,b_mn", [(0, 0), (1, 1), (0, 1), (1, 0)])
@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (300, 520, 200), (1024, 1024, 1024),
                                   (64, 16, 8), (129, 257, 136)])
@pytest.mark.parametrize("with_bias", [False, True])
def test_tc_gemm_matches_torch(a_mn, b_mn, M, N, K, with_bias, cuda_device):
    lbuild.build()
    g = torch.Generator(device="cpu").manual_seed(M * 7 + N * 3 + K)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16)
    Bt = torch.randn(N, K, generator=g).to(torch.bfloat16)
    bias = torch.randn(N, generator=g).to(torch.bfloat16) if with_bias else None
    ref = A.float() @ Bt.float().T
    if bias is not None:
        ref += bias.float()
    # storage of each operand in the requested majorness, with padded strides
    lda_pad = 8 if K % 8 == 0 else 8 - K % 8
    rnd8 = lambda v: (v + 7) // 8 * 8 + 8
    if a_mn:
        Ad = torch.zeros(K, rnd8(M), dtype=torch.bfloat16)
        Ad[:, :M] = A.T
    else:
        Ad = torch.zeros(M, K + lda_pad, dtype=torch.bfloat16)
        Ad[:, :K] = A
    if b_mn:
        Bd = torch.zeros(K, rnd8(N), dtype=torch.bfloat16)
        Bd[:, :N] = Bt.T
    else:
        Bd = torch.zeros(N, K + lda_pad, dtype=torch.bfloat16)
        Bd[:, :K] = Bt
    Ad, Bd = Ad.to(cuda_device), Bd.to(cuda_device)
    C = torch.full((M, N + 4), float("nan"), device=cuda_device)
    ws = torch.zeros(256, dtype=torch.uint8, device=cuda_device)
    rc = L.test_tc_gemm(M, N, K, Ad, Ad.shape[1], a_mn, Bd, Bd.shape[1], b_mn,
                        bias.to(cuda_device) if bias is not None else None, C, C.shape[1], ws)
    assert rc == 0
    torch.cuda.synchronize()
    assert L.lstm_status(ws) == 0
    out = C[:, :N].cpu()
    assert torch.isnan(C[:, N:]).all(), "wrote outside the output columns"
    err = (out - ref).abs().max().item() / max(ref.abs().max().item(), 1e-30)
    assert err < 1e-5, err
