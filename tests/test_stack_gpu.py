"""Stacked LSTM layers (lstm_stack_fwd / lstm_stack_bwd: the multi-layer LSTM
module of the "cmu 10-414 HW4" page, "Stack Multiple RNN Cells" of the
"mxnet-lstm" page) through the C ABI against the fp64 stacked oracle, element
by element, on the kernel paths of the layers (per-step kernels, the fused
forward and the TMEM-weight backward in one launch and in chunks, with the
layer-0 input width differing from H, and the forward as a layer wavefront),
in every compute type, and with the options; plus three identities: one layer
is the single-layer call, L layers are L single-layer calls with dx rounded
to the compute type in between, and the layer wavefront in time chunks is the
same wavefront with each layer in one launch, bit for bit.  Tolerance as in the other parity tests."""
import numpy as np
import pytest
import torch

import oracle
from backward_lstm_fwd_b200 import binding as L
from backward_lstm_fwd_b200 import synth
from tests.parity_util import assert_within, rel_err

pytestmark = pytest.mark.gpu


def stack_inputs(T, B, I, H, Lc, dt, seed):
    """Layer 0 from the workload generator; the upper layers' W, b, h0, c0,
    dhT, dcT from the generator of a workload with I = H (another seed each)."""
    layers = [synth.make_inputs(synth.custom(T, B, I if l == 0 else H, H, dt, seed=seed + 7 * l))
              for l in range(Lc)]
    inp = dict(x=layers[0]["x"], dy=layers[-1]["dy"])
    inp["W"] = [p["W"] for p in layers]
    inp["b"] = [p["b"] for p in layers]
    for k in ("h0", "c0", "dhT", "dcT"):
        inp[k] = torch.stack([p[k] for p in layers]).contiguous()
    return inp


def run_gpu_stack(inp, dev, **opt):
    Lc = len(inp["W"])
    d = {k: ([t.to(dev) for t in v] if isinstance(v, list) else v.to(dev))
         for k, v in inp.items()}
    mk = opt.pop("mask", None)
    if mk is not None:
        mk = mk.to(dev)
    st = L.forward_stack(d["x"], d["W"], d["b"], d["h0"], d["c0"], mask=mk, **opt)
    g = L.backward_stack(st, d["x"], d["W"], d["h0"], d["c0"], d["dy"], d["dhT"], d["dcT"],
                         mask=mk, **opt)
    torch.cuda.synchronize()
    n = lambda t: t.float().cpu().double().numpy()
    return dict(y=n(st.y), hT=n(st.hT), cT=n(st.cT), dx=n(g.dx), dh0=n(g.dh0), dc0=n(g.dc0),
                dW=[n(t) for t in g.dW], db=[n(t) for t in g.db], L=Lc)


def run_oracle_stack(inp, mask=None, reverse=False, gate_order="ifjo"):
    f64 = lambda t: t.double().numpy()
    Lc = len(inp["W"])
    Ws, bs = [f64(w) for w in inp["W"]], [f64(b) for b in inp["b"]]
    h0s, c0s = [f64(inp["h0"][l]) for l in range(Lc)], [f64(inp["c0"][l]) for l in range(Lc)]
    dhTs, dcTs = [f64(inp["dhT"][l]) for l in range(Lc)], [f64(inp["dcT"][l]) for l in range(Lc)]
    opt = dict(mask=None if mask is None else f64(mask), reverse=reverse,
               ijfo=gate_order == "ijfo")
    f = oracle.lstm_stack_fwd(f64(inp["x"]), Ws, bs, h0s, c0s, **opt)
    g = oracle.lstm_stack_bwd(f64(inp["x"]), Ws, h0s, c0s, f, f64(inp["dy"]), dhTs, dcTs, **opt)
    return dict(y=np.stack([fl["y"] for fl in f]), hT=np.stack([fl["hT"] for fl in f]),
                cT=np.stack([fl["cT"] for fl in f]), dx=g[0]["dx"],
                dh0=np.stack([gl["dh0"] for gl in g]), dc0=np.stack([gl["dc0"] for gl in g]),
                dW=[gl["dW"] for gl in g], db=[gl["db"] for gl in g])


def check(gpu, ref, dt, label):
    errs = {k: rel_err(gpu[k], ref[k]) for k in ("y", "hT", "cT", "dx", "dh0", "dc0")}
    for l in range(gpu["L"]):
        errs[f"dW{l}"] = rel_err(gpu["dW"][l], ref["dW"][l])
        errs[f"db{l}"] = rel_err(gpu["db"][l], ref["db"][l])
    assert_within(errs, dt, label)


CASES = [
    (6, 4, 24, 40, 3, "fp32"),      # per-step kernels, three layers
    (7, 5, 37, 48, 2, "bf16"),      # per-step kernels, bf16
    (12, 48, 64, 512, 2, "bf16"),   # TMEM-weight kernels, layer 0 narrower than H
    (40, 64, 1024, 512, 2, "bf16"), # chunked backward, layer 0 wider than H
    (12, 48, 64, 512, 3, "fp16"),   # fp16
    (6, 128, 64, 512, 2, "bf16"),   # the forward with two batch streams per cluster
    (64, 64, 256, 512, 2, "bf16"),  # the forward as a layer wavefront (8 chunks of 8 steps)
]


@pytest.mark.parametrize("case", CASES)
def test_stack(case, cuda_device):
    T, B, I, H, Lc, dt = case
    inp = stack_inputs(T, B, I, H, Lc, dt, seed=T + B + H)
    gpu = run_gpu_stack(inp, cuda_device)
    ref = run_oracle_stack(inp)
    check(gpu, ref, dt, f"stack {case}")


# (T, B, I, H, L, dtype, reverse, gate order, chunks per layer)
WAVE_CASES = [
    (64, 64, 512, 512, 2, "bf16", False, "ifjo", 8),
    (43, 64, 1024, 512, 3, "fp16", False, "ifjo", 5),  # chunks of 8 or 9 steps
    (40, 128, 256, 512, 2, "bf16", True, "ijfo", 5),   # reverse direction
]


@pytest.mark.parametrize("case", WAVE_CASES)
def test_stack_wavefront_chunks_are_seamless(case, cuda_device, monkeypatch):
    """The layer wavefront runs each layer in time chunks on its own stream, a
    layer's chunk after the same chunk of the layer below.  A chunk continues
    its layer from the saved h (the compute type, as the kernel reads h_{t-1}
    every step) and c (fp32, the value the kernel keeps in registers) of the
    step before it, so the chunked run gives the bits of each layer in one
    launch (LSTM_STACK_CHUNKS=1, the same grids); with the wavefront off, the
    layers run one after another on the full-device plan, whose summation
    order differs, and the stack matches the oracle either way."""
    T, B, I, H, Lc, dt, reverse, order, nch = case
    inp = stack_inputs(T, B, I, H, Lc, dt, seed=T + Lc)
    d = {k: ([t.to(cuda_device) for t in v] if isinstance(v, list) else v.to(cuda_device))
         for k, v in inp.items()}
    outs = {}
    for label, env, want in (("chunked", {}, nch), ("one launch", {"LSTM_STACK_CHUNKS": "1"}, 1),
                             ("layer by layer", {"LSTM_STACK_WAVE": "0"}, 0)):
        monkeypatch.delenv("LSTM_STACK_CHUNKS", raising=False)
        monkeypatch.delenv("LSTM_STACK_WAVE", raising=False)
        for k, v in env.items():
            monkeypatch.setenv(k, v)
        outs[label] = L.forward_stack(d["x"], d["W"], d["b"], d["h0"], d["c0"], reverse=reverse,
                                      gate_order=order)
        torch.cuda.synchronize()
        assert L.test_last_stack_chunks()[0] == want, label
    a, b = outs["chunked"], outs["one launch"]
    for k in ("y", "hT", "cT", "gates", "cells"):
        assert torch.equal(getattr(a, k), getattr(b, k)), k
    # the chunked wavefront, and the backward on its saved state, against the oracle
    g = L.backward_stack(a, d["x"], d["W"], d["h0"], d["c0"], d["dy"], d["dhT"], d["dcT"],
                         reverse=reverse, gate_order=order)
    torch.cuda.synchronize()
    n = lambda t: t.float().cpu().double().numpy()
    gpu = dict(y=n(a.y), hT=n(a.hT), cT=n(a.cT), dx=n(g.dx), dh0=n(g.dh0), dc0=n(g.dc0),
               dW=[n(t) for t in g.dW], db=[n(t) for t in g.db], L=Lc)
    check(gpu, run_oracle_stack(inp, reverse=reverse, gate_order=order), dt,
          f"stack wavefront {case}")
    seq = outs["layer by layer"]
    errs = {k: rel_err(getattr(a, k).float().cpu().double().numpy(),
                       getattr(seq, k).float().cpu().double().numpy())
            for k in ("y", "hT", "cT")}
    assert_within(errs, dt, f"wavefront vs layer by layer {case}")


# (T, B, I, H, L, dtype, reverse, gate order, backward chunks per layer)
WAVE_BWD_CASES = [
    (64, 64, 512, 512, 2, "bf16", False, "ifjo", 4),
    (48, 64, 1024, 512, 3, "fp16", False, "ifjo", 3),
    (40, 128, 256, 512, 2, "bf16", True, "ijfo", 2),   # reverse direction
]


@pytest.mark.parametrize("case", WAVE_BWD_CASES)
def test_stack_backward_wavefront_equals_layer_by_layer(case, cuda_device):
    """The backward layer wavefront runs each layer's reverse-time chunks on a
    stream of its own; after a chunk, the dx GEMM over its rows and the
    rounding to the compute type give the lower layer the dy of the same
    chunk, which its chunk waits for.  The chunks, kernels, GEMM tiles and
    accumulation order are those of the layer-by-layer backward, so dx, dW,
    dh0 and dc0 are the same bits; db, whose batch sum runs per batch group,
    follows the wavefront's grid (half the co-resident clusters per layer)
    in its order of additions.  The layer-by-layer run here is the fallback a
    caller gets from a workspace smaller than the wavefront's (but at least the
    layer-by-layer size); both match the oracle (the first case through the
    oracle cases of CASES, the others here)."""
    T, B, I, H, Lc, dt, reverse, order, nch = case
    inp = stack_inputs(T, B, I, H, Lc, dt, seed=3 * T + Lc)
    d = {k: ([t.to(cuda_device) for t in v] if isinstance(v, list) else v.to(cuda_device))
         for k, v in inp.items()}
    st = L.forward_stack(d["x"], d["W"], d["b"], d["h0"], d["c0"], reverse=reverse,
                         gate_order=order)
    full = L.stack_bwd_workspace_size(st.dims, Lc)
    least = L.stack_bwd_workspace_size_min(st.dims, Lc)
    assert least < full
    grads = {}
    for label, nbytes, want in (("wavefront", full, nch), ("layer by layer", full - 1, 0),
                                ("smallest", least, 0)):
        ws = L.empty_workspace(nbytes, cuda_device)[:nbytes]
        grads[label] = L.backward_stack(st, d["x"], d["W"], d["h0"], d["c0"], d["dy"], d["dhT"],
                                        d["dcT"], ws=ws, reverse=reverse, gate_order=order)
        torch.cuda.synchronize()
        assert L.test_last_stack_chunks()[1] == want, label
    a = grads["wavefront"]
    for b in (grads["layer by layer"], grads["smallest"]):
        for k in ("dx", "dh0", "dc0"):
            assert torch.equal(getattr(a, k), getattr(b, k)), k
        for l in range(Lc):
            assert torch.equal(a.dW[l], b.dW[l]), l
            # db adds its batch rows per batch group of the plan, then the
            # groups: the order (not the terms) follows the grid
            torch.testing.assert_close(a.db[l], b.db[l], rtol=1e-5, atol=1e-5)
    if case != WAVE_BWD_CASES[0]:
        n = lambda t: t.float().cpu().double().numpy()
        gpu = dict(y=n(st.y), hT=n(st.hT), cT=n(st.cT), dx=n(a.dx), dh0=n(a.dh0), dc0=n(a.dc0),
                   dW=[n(t) for t in a.dW], db=[n(t) for t in a.db], L=Lc)
        check(gpu, run_oracle_stack(inp, reverse=reverse, gate_order=order), dt,
              f"stack backward wavefront {case}")


def test_stack_with_options(cuda_device):
    T, B, I, H, Lc, dt = 40, 64, 96, 512, 2, "bf16"
    inp = stack_inputs(T, B, I, H, Lc, dt, seed=5)
    mask = synth.length_mask(T, B, H, synth.random_lengths(T, B, seed=3), dt)
    gpu = run_gpu_stack(inp, cuda_device, mask=mask, reverse=True, gate_order="ijfo")
    ref = run_oracle_stack(inp, mask=mask, reverse=True, gate_order="ijfo")
    check(gpu, ref, dt, "stack, mask, reverse, ijfo")


def test_one_layer_stack_is_the_single_layer_call(cuda_device):
    T, B, I, H = 12, 48, 64, 512
    inp = stack_inputs(T, B, I, H, 1, "bf16", seed=1)
    d = {k: ([t.to(cuda_device) for t in v] if isinstance(v, list) else v.to(cuda_device))
         for k, v in inp.items()}
    st = L.forward_stack(d["x"], d["W"], d["b"], d["h0"], d["c0"])
    g = L.backward_stack(st, d["x"], d["W"], d["h0"], d["c0"], d["dy"], d["dhT"], d["dcT"])
    s1 = L.forward(d["x"], d["W"][0], d["b"][0], d["h0"][0], d["c0"][0])
    g1 = L.backward(s1, d["x"], d["W"][0], d["h0"][0], d["c0"][0], d["dy"], d["dhT"][0],
                    d["dcT"][0])
    torch.cuda.synchronize()
    assert torch.equal(st.y[0], s1.y) and torch.equal(st.cT[0], s1.cT)
    assert torch.equal(g.dx, g1.dx) and torch.equal(g.dW[0], g1.dW)
    assert torch.equal(g.db[0], g1.db) and torch.equal(g.dh0[0], g1.dh0)


@pytest.mark.parametrize("dt", ["bf16", "fp32"])
def test_stack_is_composed_single_layer_calls(dt, cuda_device):
    """The host loop adds nothing: the same layers run as separate calls, with
    the upper layer's dx rounded to the compute type by torch, give the same
    bits."""
    T, B, I, H, Lc = 9, 32, 48, 256, 3
    inp = stack_inputs(T, B, I, H, Lc, dt, seed=8)
    d = {k: ([t.to(cuda_device) for t in v] if isinstance(v, list) else v.to(cuda_device))
         for k, v in inp.items()}
    st = L.forward_stack(d["x"], d["W"], d["b"], d["h0"], d["c0"])
    g = L.backward_stack(st, d["x"], d["W"], d["h0"], d["c0"], d["dy"], d["dhT"], d["dcT"])
    xs, states = [d["x"]], []
    for l in range(Lc):
        s = L.forward(xs[-1], d["W"][l], d["b"][l], d["h0"][l], d["c0"][l])
        states.append(s)
        xs.append(s.y)
    up, grads = d["dy"], [None] * Lc
    for l in reversed(range(Lc)):
        grads[l] = L.backward(states[l], xs[l], d["W"][l], d["h0"][l], d["c0"][l], up,
                              d["dhT"][l], d["dcT"][l])
        up = grads[l].dx.to(synth.torch_dtype(dt))
    torch.cuda.synchronize()
    for l in range(Lc):
        assert torch.equal(st.y[l], states[l].y), l
        assert torch.equal(st.hT[l], states[l].hT) and torch.equal(st.cT[l], states[l].cT), l
        assert torch.equal(g.dW[l], grads[l].dW) and torch.equal(g.db[l], grads[l].db), l
        assert torch.equal(g.dh0[l], grads[l].dh0) and torch.equal(g.dc0[l], grads[l].dc0), l
    assert torch.equal(g.dx, grads[0].dx)


@pytest.mark.parametrize("dt", ["fp32", "bf16"])
def test_stack_empty_sequence(dt, cuda_device):
    """T = 0: no layer steps; every layer's final state is its initial state and
    the gradients at the initial states are the ones given at the final states."""
    T, B, I, H, Lc = 0, 8, 16, 32, 2
    inp = stack_inputs(T, B, I, H, Lc, dt, seed=4)
    gpu = run_gpu_stack(inp, cuda_device)
    for l in range(Lc):
        np.testing.assert_array_equal(gpu["hT"][l], inp["h0"][l].double().numpy())
        np.testing.assert_array_equal(gpu["cT"][l], inp["c0"][l].double().numpy())
        np.testing.assert_array_equal(gpu["dh0"][l], inp["dhT"][l].double().numpy())
        np.testing.assert_array_equal(gpu["dc0"][l], inp["dcT"][l].double().numpy())
        assert not gpu["dW"][l].any() and not gpu["db"][l].any()
