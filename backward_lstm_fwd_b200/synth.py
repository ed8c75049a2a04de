"""Seeded synthetic inputs for the LSTM forward + BPTT path.

This module holds random draws, casts and indexing only -- none of the LSTM
arithmetic -- so that the CUDA library's tests and the fp64 oracle can be fed
the very same values.

Distributions follow the pages' workloads: weights and bias uniform in
(-1/sqrt(H), 1/sqrt(H)) (the U(-sqrt(k), sqrt(k)), k = 1/hidden_size rule of the
torch.ao.nn.quantized.dynamic.GRU page and of the CMU 10-414 LSTM notes),
x uniform in (-1, 1), initial states N(0, 0.5^2), upstream gradients N(0, 1).

Draw order (one torch CPU generator seeded per workload, all in fp32):
  W[4H, H+I], b[4H], x[T, B, I], h0[B, H], c0[B, H], dy[T, B, H],
  then dhT[B, H] and dcT[B, H] only for workloads that carry them
  (otherwise both are zero and nothing is drawn).
For bf16 (fp16) workloads x, W, b, h0, dy and dhT are rounded to bf16 (fp16)
after the draw; c0 and dcT stay fp32 (the cell state is fp32 throughout).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional, Sequence

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int
    B: int
    I: int
    H: int
    dtype: str            # "fp32", "bf16" or "fp16": the type x, W, b, h0, dy, y, gates are stored in
    seed: int
    dhdc: bool            # draw dhT / dcT (else zeros)
    dy_last: Optional[int] = None  # keep dy only on the last dy_last steps

    @property
    def rows(self) -> int:
        return self.T * self.B

    @property
    def flops(self) -> float:
        """Algorithmic FLOPs of forward + backward: 24 * H * (H + I) per (t, b) row
        (gate pre-activations, delta z, and dW; 2 * 4H * (H + I) each)."""
        return 24.0 * self.H * (self.H + self.I) * self.rows


WORKLOADS: Dict[str, Workload] = {w.name: w for w in [
    Workload("lstm_T8_B2_I16_H32_fp32", 8, 2, 16, 32, "fp32", 0, False),
    Workload("lstm_T64_B32_I256_H256_fp32", 64, 32, 256, 256, "fp32", 1, True),
    Workload("lstm_T128_B64_I512_H512_bf16", 128, 64, 512, 512, "bf16", 2, False),
    Workload("lstm_T256_B128_I1024_H1024_bf16", 256, 128, 1024, 1024, "bf16", 3, True),
    Workload("lstm_T1024_B16_I256_H1024_bf16", 1024, 16, 256, 1024, "bf16", 4, True, dy_last=64),
]}

# The large-batch throughput workload that bench.py times.
BENCH_WORKLOAD = "lstm_T256_B128_I1024_H1024_bf16"


def custom(T: int, B: int, I: int, H: int, dtype: str, seed: int = 123,
           dhdc: bool = True, dy_last: Optional[int] = None) -> Workload:
    return Workload(f"lstm_T{T}_B{B}_I{I}_H{H}_{dtype}_s{seed}", T, B, I, H, dtype, seed,
                    dhdc, dy_last)


def torch_dtype(dtype: str) -> torch.dtype:
    return {"fp32": torch.float32, "bf16": torch.bfloat16, "fp16": torch.float16}[dtype]


def make_inputs(w: Workload) -> Dict[str, torch.Tensor]:
    """Draw the workload's inputs on the CPU (contiguous tensors)."""
    g = torch.Generator().manual_seed(w.seed)
    T, B, I, H = w.T, w.B, w.I, w.H
    bound = 1.0 / math.sqrt(H) if H > 0 else 0.0

    def unif(shape, lo, hi):
        return torch.rand(shape, generator=g, dtype=torch.float32) * (hi - lo) + lo

    W = unif((4 * H, H + I), -bound, bound)
    b = unif((4 * H,), -bound, bound)
    x = unif((T, B, I), -1.0, 1.0)
    h0 = torch.randn((B, H), generator=g, dtype=torch.float32) * 0.5
    c0 = torch.randn((B, H), generator=g, dtype=torch.float32) * 0.5
    dy = torch.randn((T, B, H), generator=g, dtype=torch.float32)
    if w.dhdc:
        dhT = torch.randn((B, H), generator=g, dtype=torch.float32)
        dcT = torch.randn((B, H), generator=g, dtype=torch.float32)
    else:
        dhT = torch.zeros((B, H), dtype=torch.float32)
        dcT = torch.zeros((B, H), dtype=torch.float32)
    if w.dy_last is not None and w.dy_last < T:
        dy[: T - w.dy_last] = 0.0
    cd = torch_dtype(w.dtype)
    return dict(x=x.to(cd).contiguous(), W=W.to(cd).contiguous(), b=b.to(cd).contiguous(),
                h0=h0.to(cd).contiguous(), c0=c0.contiguous(), dy=dy.to(cd).contiguous(),
                dhT=dhT.to(cd).contiguous(), dcT=dcT.contiguous())


def select_sequences(inputs: Dict[str, torch.Tensor], idx: Sequence[int]) -> Dict[str, torch.Tensor]:
    """The sub-batch made of sequences ``idx`` (sequences are independent)."""
    ix = torch.as_tensor(list(idx), dtype=torch.long)
    out = {}
    for k, v in inputs.items():
        if k in ("x", "dy", "mask"):
            out[k] = v.index_select(1, ix).contiguous()
        elif k in ("h0", "c0", "dhT", "dcT"):
            out[k] = v.index_select(0, ix).contiguous()
        else:
            out[k] = v
    return out


def as_float64(inputs: Dict[str, torch.Tensor]):
    """Exact widening of every input to float64 numpy arrays (what the oracle reads)."""
    return {k: v.double().numpy() for k, v in inputs.items()}


# ------------------------------------------------------------- variable length
def random_lengths(T: int, B: int, seed: int) -> list:
    """Per-sequence lengths in 0..T, seeded; the first three sequences (when
    there are that many) take the edge lengths T, 0 and 1."""
    g = torch.Generator().manual_seed(seed)
    lengths = torch.randint(0, T + 1, (B,), generator=g).tolist()
    for n, L in enumerate([T, 0, 1][:B]):
        lengths[n] = min(L, T)
    return lengths


def length_mask(T: int, B: int, H: int, lengths, dtype: str) -> torch.Tensor:
    """Mask [T][B][H] with 1 on the first lengths[n] steps of sequence n and 0
    on the padding after them (the seq_length input, in the compute type)."""
    m = torch.zeros(T, B, H)
    for n, L in enumerate(lengths):
        m[:L, n, :] = 1.0
    return m.to(torch_dtype(dtype)).contiguous()


def random_mask(T: int, B: int, H: int, dtype: str, seed: int, p_pad: float = 0.3) -> torch.Tensor:
    """Element-wise random 0/1 mask [T][B][H] (padding with probability p_pad)."""
    g = torch.Generator().manual_seed(seed)
    m = (torch.rand(T, B, H, generator=g) >= p_pad).float()
    return m.to(torch_dtype(dtype)).contiguous()
