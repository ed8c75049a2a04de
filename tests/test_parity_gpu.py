"""CUDA path vs the fp64 oracle, element by element, through the C ABI.

Full-size runs of the five workloads on the whole batch (the launch
configuration bench.py times), a long sequence with upstream gradient on every step,
odd shapes that leave ragged tiles, and the degenerate cases (empty sequence or
batch, no input features, absent optional inputs).  Tolerance per output
tensor: max|gpu - ref| / max|ref| <= 1e-4 (fp32), 2e-2 (bf16) or 2.5e-3 (fp16)."""
import numpy as np
import pytest
import torch

from backward_lstm_fwd_b200 import binding as L
from backward_lstm_fwd_b200 import synth
from tests.parity_util import OUTS, assert_within, compare, run_gpu, run_oracle

pytestmark = pytest.mark.gpu

# The five workloads, full size, every output tensor against the oracle on the
# whole batch (the two largest take the oracle about 20-40 s on 16 host cores).
FULL = ["lstm_T8_B2_I16_H32_fp32", "lstm_T64_B32_I256_H256_fp32", "lstm_T128_B64_I512_H512_bf16",
        "lstm_T256_B128_I1024_H1024_bf16", "lstm_T1024_B16_I256_H1024_bf16"]


# recurrent kernel each workload must run on (see lstm_test_last_paths)
EXPECTED_PATHS = {"lstm_T8_B2_I16_H32_fp32": (5, 5), "lstm_T64_B32_I256_H256_fp32": (5, 5),
                  "lstm_T128_B64_I512_H512_bf16": (3, 4),
                  "lstm_T256_B128_I1024_H1024_bf16": (3, 4),
                  "lstm_T1024_B16_I256_H1024_bf16": (3, 3)}


@pytest.mark.parametrize("name", FULL)
def test_workload_full(name, cuda_device):
    w = synth.WORKLOADS[name]
    inp = synth.make_inputs(w)
    gpu = run_gpu(inp, cuda_device)
    assert L.test_last_paths() == EXPECTED_PATHS[name]
    ref = run_oracle(inp)
    errs = compare(gpu, ref, w.dtype, OUTS + ("gates", "cells"))
    assert_within(errs, w.dtype, name)


def test_long_sequence_dense_upstream(cuda_device):
    """The T = 1024, B = 16, I = 256, H = 1024 shape with dy drawn on every
    step: dh0 and dc0 are then O(1), so the whole 1024-step delta h / delta c
    carry down to t = 0 is checked at the bf16 tolerance (the workload itself
    has dy only on its last 64 steps, which leaves dh0 / dc0 near 1e-189)."""
    w = synth.custom(1024, 16, 256, 1024, "bf16", seed=41)
    inp = synth.make_inputs(w)
    gpu = run_gpu(inp, cuda_device)
    assert L.test_last_paths() == (3, 3)  # 16 rows: one batch stream
    ref = run_oracle(inp)
    for k in ("dh0", "dc0"):
        assert float(np.max(np.abs(ref[k]))) > 1e-3, (k, float(np.max(np.abs(ref[k]))))
    assert_within(compare(gpu, ref, "bf16", OUTS + ("gates", "cells")), "bf16", w.name)


ODD = [
    (5, 3, 37, 45, "fp32"), (1, 1, 1, 1, "fp32"), (3, 67, 100, 72, "fp32"),
    (2, 130, 64, 128, "fp32"), (7, 5, 16, 33, "fp32"),
    (5, 3, 37, 45, "bf16"), (1, 1, 1, 1, "bf16"), (3, 67, 100, 72, "bf16"),
    (4, 130, 128, 128, "bf16"), (9, 16, 64, 64, "bf16"), (3, 200, 192, 256, "bf16"),
    # backward with the weights in tensor memory: two ragged batch groups,
    # an odd count of unit slices, and the largest H whose K slice fits TMEM
    (5, 200, 96, 512, "bf16"), (3, 37, 64, 640, "bf16"), (2, 16, 32, 1536, "bf16"),
    # the backward in reverse-time chunks with dW / dx of each chunk beside the
    # next one: 37 steps in 2 chunks, chunk row counts off the 64-row K blocks
    (37, 200, 96, 512, "bf16"),
    # W rows of H + I elements off the 16-byte grid, with H on the unit grids
    # of the tensor-map recurrences: those must step aside for the per-step kernels
    (4, 6, 37, 48, "bf16"), (4, 6, 37, 64, "bf16"),
    # the forward with two batch streams per cluster at its shortest sequences
    (1, 200, 96, 512, "bf16"), (2, 100, 64, 1024, "bf16"),
    # the backward with two batch streams per group: a ragged last stream
    # (rows 112..119 of 4 groups of 32), a ragged second stream of one group
    # of 128, and H = 1536, whose 12 K chunks per step wrap around an
    # 8-stage ring per stream
    (5, 120, 96, 512, "bf16"), (3, 100, 64, 1024, "bf16"), (3, 64, 64, 1536, "bf16"),
]


# recurrent kernels of the odd bf16 shapes above (see lstm_test_last_paths):
# the forward with the input projection fused wherever H is a multiple of 32
# (clusters of 4, 2 and 1 among these), the backward with the weights in TMEM,
# keyed by (B, H)
ODD_FWD_PATH = {64: 3, 128: 3, 256: 3, 512: 3, 640: 3, 1024: 3, 1536: 3}
ODD_BWD_PATH = {(200, 512): 3, (37, 640): 3, (16, 1536): 3, (120, 512): 4, (100, 1024): 4,
                (64, 1536): 4}


@pytest.mark.parametrize("T,B,I,H,dt", ODD)
def test_odd_shapes(T, B, I, H, dt, cuda_device):
    w = synth.custom(T, B, I, H, dt, seed=T * 1000 + B + I + H)
    inp = synth.make_inputs(w)
    gpu = run_gpu(inp, cuda_device)
    if dt == "bf16" and I % 8 != 0:  # no tensor-map forward recurrence
        assert L.test_last_paths()[0] == 5
    elif dt == "bf16" and H in ODD_FWD_PATH:
        assert L.test_last_paths()[0] == ODD_FWD_PATH[H]
    if dt == "bf16" and (B, H) in ODD_BWD_PATH:
        assert L.test_last_paths()[1] == ODD_BWD_PATH[(B, H)]
    ref = run_oracle(inp)
    assert_within(compare(gpu, ref, dt), dt, w.name)


@pytest.mark.parametrize("dt,B,I,H", [("fp32", 4, 24, 40), ("bf16", 4, 24, 40), ("fp16", 4, 24, 40),
                                      ("bf16", 128, 64, 512)])
def test_optional_inputs_absent(dt, B, I, H, cuda_device):
    """Also at B = 128, H = 512: the fused forward with two batch streams
    starts from h0 = 0 without loading it."""
    w = synth.custom(6, B, I, H, dt, seed=5)
    inp = synth.make_inputs(w)
    drop = ("b", "h0", "c0", "dhT", "dcT")
    gpu = run_gpu(inp, cuda_device, drop=drop)
    ref = run_oracle(inp, drop=drop)
    assert_within(compare(gpu, ref, dt), dt, "optional inputs NULL")
    drop = ("dy",)
    gpu = run_gpu(inp, cuda_device, drop=drop)
    ref = run_oracle(inp, drop=drop)
    assert_within(compare(gpu, ref, dt), dt, "dy NULL")


@pytest.mark.parametrize("dt", ["fp32", "bf16", "fp16"])
def test_empty_sequence(dt, cuda_device):
    w = synth.custom(0, 3, 8, 16, dt, seed=2)
    inp = synth.make_inputs(w)
    gpu = run_gpu(inp, cuda_device)
    np.testing.assert_array_equal(gpu["hT"], inp["h0"].double().numpy())
    np.testing.assert_array_equal(gpu["cT"], inp["c0"].double().numpy())
    np.testing.assert_array_equal(gpu["dh0"], inp["dhT"].double().numpy())
    np.testing.assert_array_equal(gpu["dc0"], inp["dcT"].double().numpy())
    assert not gpu["dW"].any() and not gpu["db"].any()


@pytest.mark.parametrize("dt", ["fp32", "bf16", "fp16"])
def test_empty_batch_and_no_inputs(dt, cuda_device):
    gpu = run_gpu(synth.make_inputs(synth.custom(4, 0, 8, 16, dt)), cuda_device)
    assert gpu["y"].shape == (4, 0, 16)
    assert not gpu["dW"].any() and not gpu["db"].any()
    w = synth.custom(4, 3, 0, 16, dt, seed=9)
    inp = synth.make_inputs(w)
    assert_within(compare(run_gpu(inp, cuda_device), run_oracle(inp), dt), dt, "I = 0")


@pytest.mark.parametrize("shape", [(12, 8, 64, 64, "bf16"), (16, 32, 64, 256, "fp32")])
def test_side_stream_and_repeat(shape, cuda_device):
    """Calls are ordered on the stream they are given, and a second call with
    the same workspace gives the same bits.  The fp32 case runs the K-split
    persistent recurrences, dW split into two row slabs, and db and dx on the
    library's auxiliary streams, joined back into the caller's side stream."""
    T, B, I, H, dt = shape
    w = synth.custom(T, B, I, H, dt, seed=3)
    inp = synth.make_inputs(w)
    s = torch.cuda.Stream()
    a = run_gpu(inp, cuda_device, stream=s)
    b = run_gpu(inp, cuda_device, stream=s)
    for k in OUTS:
        np.testing.assert_array_equal(a[k], b[k])
    assert_within(compare(a, run_oracle(inp), dt), dt, "side stream")



@pytest.mark.parametrize("chunks", ["1", "3", "5"])
@pytest.mark.parametrize("B,path", [(40, 3), (64, 4)])
def test_backward_chunk_counts(chunks, B, path, cuda_device, monkeypatch):
    """The backward in 1 (one launch, no overlap), 3 or 5 reverse-time chunks
    (dW / dx of each chunk beside the next one) gives the oracle's gradients,
    with one batch stream per group (B = 40) and with two (B = 64)."""
    monkeypatch.setenv("LSTM_BWD_CHUNKS", chunks)
    w = synth.custom(41, B, 64, 512, "bf16", seed=17)
    inp = synth.make_inputs(w)
    gpu = run_gpu(inp, cuda_device)
    assert L.test_last_paths() == (3, path)
    assert_within(compare(gpu, run_oracle(inp), "bf16"), "bf16", f"{chunks} chunks")


@pytest.mark.parametrize("shape", [(20, 128, 64, 1024), (33, 64, 96, 512)])
def test_two_stream_backward_equals_one_stream(shape, cuda_device, monkeypatch):
    """The backward with two decoupled batch streams per group computes every
    element in the same order as the one-stream kernel: the same bits."""
    T, B, I, H = shape
    w = synth.custom(T, B, I, H, "bf16", seed=T + B)
    inp = synth.make_inputs(w)
    two = run_gpu(inp, cuda_device)
    fwd_path = L.test_last_paths()[0]
    assert L.test_last_paths()[1] == 4
    monkeypatch.setenv("LSTM_BWD_STREAMS", "1")
    one = run_gpu(inp, cuda_device)
    assert L.test_last_paths() == (fwd_path, 3)
    for k in ("dx", "dW", "db", "dh0", "dc0"):
        np.testing.assert_array_equal(two[k], one[k], err_msg=k)



@pytest.mark.parametrize("ks", [1, 2, 4, 8])
@pytest.mark.parametrize("shape", [(12, 32, 256, 256, "fp32"), (6, 130, 64, 128, "fp32"),
                                   (7, 5, 37, 45, "bf16"), (5, 17, 40, 100, "fp16"),
                                   (1, 32, 64, 256, "fp32")])
def test_persistent_k_split_cluster_sizes(shape, ks, cuda_device, monkeypatch):
    """Each cluster size of the persistent CUDA-core recurrences' K split (KS
    CTAs per cluster, each contracting one K slice, the partial sums sent to
    the CTA that finishes their units by DSMEM copies) against the oracle,
    forward and backward; a size that does not fit the shape leaves the
    per-step kernels to run."""
    T, B, I, H, dt = shape
    w = synth.custom(T, B, I, H, dt, seed=T * 11 + ks)
    inp = synth.make_inputs(w)
    monkeypatch.setenv("LSTM_PERSIST_KS", str(ks))
    out = run_gpu(inp, cuda_device, reverse=ks == 4)
    fp, bp = L.test_last_paths()
    fk, bk = L.test_last_persist_split()
    assert fp in (0, 5) and bp in (0, 5)
    if fp == 5:
        assert fk == ks
    if bp == 5:
        assert bk == ks
    if ks == 1:
        assert (fp, bp) == (5, 5)
    if ks == 8 and H == 256:
        assert bp == 5  # 8 clusters of 8 (the forward's 16 need not be co-resident)
    ref = run_oracle(inp, reverse=ks == 4)
    assert_within(compare(out, ref, dt, OUTS + ("gates", "cells")), dt,
                  f"{w.name} persistent KS={ks}")


@pytest.mark.parametrize("shape", [(64, 32, 256, 256, "fp32"), (9, 6, 24, 40, "fp32"),
                                   (7, 5, 37, 45, "bf16"), (5, 130, 96, 1024, "fp32")])
@pytest.mark.parametrize("opts", [{}, {"reverse": True, "ijfo": True}, {"mask": True}])
def test_persistent_cuda_core_recurrences(shape, opts, cuda_device, monkeypatch):
    """The persistent CUDA-core recurrences (all steps in one launch) against
    the oracle and against the per-step kernels (LSTM_PERSIST=0): the same
    epilogues, the products summed in another order."""
    T, B, I, H, dt = shape
    w = synth.custom(T, B, I, H, dt, seed=T * 7 + H)
    inp = synth.make_inputs(w)
    kw = dict(opts)
    if kw.pop("mask", False):
        kw["mask"] = synth.length_mask(T, B, H, synth.random_lengths(T, B, seed=B + H), dt)
    per = run_gpu(inp, cuda_device, **kw)
    assert L.test_last_paths() == (5, 5)
    ref = run_oracle(inp, **kw)
    assert_within(compare(per, ref, dt, OUTS + ("gates", "cells")), dt, w.name + " persistent")
    monkeypatch.setenv("LSTM_PERSIST", "0")
    stp = run_gpu(inp, cuda_device, **kw)
    assert L.test_last_paths() == (0, 0)
    assert_within(compare(stp, ref, dt, OUTS + ("gates", "cells")), dt, w.name + " per step")
