"""The seeded input generators shared by the tests, the bench and the oracle
runs: deterministic per seed, the shapes and ranges of the workload recipe
(W, b ~ U(-1/sqrt(H), 1/sqrt(H)), x ~ U(-1, 1), states ~ N(0, 0.5^2),
upstream gradients ~ N(0, 1)), exact rounding to the compute type, and the
variable-length masks.  They hold none of the method's arithmetic."""
import math

import numpy as np
import pytest
import torch

from backward_lstm_fwd_b200 import synth


def test_workloads_are_the_five_configurations():
    w = synth.WORKLOADS
    assert set(w) == {"lstm_T8_B2_I16_H32_fp32", "lstm_T64_B32_I256_H256_fp32",
                      "lstm_T128_B64_I512_H512_bf16", "lstm_T256_B128_I1024_H1024_bf16",
                      "lstm_T1024_B16_I256_H1024_bf16"}
    assert synth.BENCH_WORKLOAD == "lstm_T256_B128_I1024_H1024_bf16"
    assert [w[k].seed for k in sorted(w, key=lambda k: w[k].seed)] == [0, 1, 2, 3, 4]


def test_deterministic_and_seed_dependent():
    w = synth.custom(5, 3, 7, 8, "fp32", seed=11)
    a, b = synth.make_inputs(w), synth.make_inputs(w)
    for k in a:
        assert torch.equal(a[k], b[k]), k
    c = synth.make_inputs(synth.custom(5, 3, 7, 8, "fp32", seed=12))
    assert not torch.equal(a["W"], c["W"])


@pytest.mark.parametrize("dt", ["fp32", "bf16", "fp16"])
def test_shapes_ranges_and_types(dt):
    T, B, I, H = 6, 4, 10, 16
    inp = synth.make_inputs(synth.custom(T, B, I, H, dt, seed=3))
    cd = synth.torch_dtype(dt)
    shapes = dict(x=(T, B, I), W=(4 * H, H + I), b=(4 * H,), h0=(B, H), c0=(B, H),
                  dy=(T, B, H), dhT=(B, H), dcT=(B, H))
    for k, s in shapes.items():
        assert tuple(inp[k].shape) == s, k
        assert inp[k].dtype == (torch.float32 if k in ("c0", "dcT") else cd), k
        assert inp[k].is_contiguous()
    bound = 1.0 / math.sqrt(H)
    tol = 1e-2 * bound  # rounding to the 16-bit types
    assert float(inp["W"].float().abs().max()) <= bound + tol
    assert float(inp["b"].float().abs().max()) <= bound + tol
    assert float(inp["x"].float().abs().max()) <= 1.0


def test_sixteen_bit_inputs_are_the_rounded_fp32_draws():
    T, B, I, H = 4, 3, 8, 8
    f = synth.make_inputs(synth.custom(T, B, I, H, "fp32", seed=5))
    for dt, cd in (("bf16", torch.bfloat16), ("fp16", torch.float16)):
        h = synth.make_inputs(synth.custom(T, B, I, H, dt, seed=5))
        for k in ("x", "W", "b", "h0", "dy", "dhT"):
            assert torch.equal(h[k], f[k].to(cd)), (dt, k)
        assert torch.equal(h["c0"], f["c0"]) and torch.equal(h["dcT"], f["dcT"])


def test_last_steps_only_upstream_gradient():
    w = synth.WORKLOADS["lstm_T1024_B16_I256_H1024_bf16"]
    small = synth.custom(12, 2, 4, 8, "bf16", seed=4, dy_last=3)
    dy = synth.make_inputs(small)["dy"].float()
    assert not dy[:9].any() and dy[9:].abs().sum() > 0
    assert w.dy_last == 64


def test_length_masks():
    T, B, H = 7, 6, 3
    lengths = synth.random_lengths(T, B, seed=9)
    assert lengths[:3] == [T, 0, 1] and all(0 <= L <= T for L in lengths)
    assert synth.random_lengths(T, B, seed=9) == lengths
    m = synth.length_mask(T, B, H, lengths, "bf16").float()
    for n, L in enumerate(lengths):
        assert m[:L, n].eq(1).all() and m[L:, n].eq(0).all()
    r = synth.random_mask(T, B, H, "fp32", seed=2)
    assert set(np.unique(r.numpy()).tolist()) <= {0.0, 1.0}


def test_select_sequences_takes_whole_sequences():
    inp = synth.make_inputs(synth.custom(3, 5, 4, 6, "fp32", seed=1))
    sub = synth.select_sequences(inp, [4, 1])
    assert torch.equal(sub["x"], inp["x"][:, [4, 1]])
    assert torch.equal(sub["h0"], inp["h0"][[4, 1]])
    assert torch.equal(sub["W"], inp["W"])
