"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
binding, run the oracle on the same (exactly widened) inputs, and compare each
output tensor by max|gpu - ref| / max|ref|."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from backward_lstm_fwd_b200 import binding as L
from backward_lstm_fwd_b200 import build as lbuild
from backward_lstm_fwd_b200 import synth

# Per-tensor tolerance on max|gpu - ref| / max|ref|: 1e-4 for the fp32 compute
# type, 2e-2 for bf16 operands with fp32 accumulation and fp32 cell state, and
# for fp16 the bf16 figure scaled by the ratio of the unit roundoffs
# (2^-11 / 2^-8): 2.5e-3.
TOL = {"fp32": 1e-4, "bf16": 2e-2, "fp16": 2.5e-3}
FWD_OUTS = ("y", "hT", "cT")
BWD_OUTS = ("dx", "dW", "db", "dh0", "dc0")
OUTS = FWD_OUTS + BWD_OUTS


FLT_MIN_NORMAL = float(np.finfo(np.float32).tiny)  # 2^-126
FLT_SUBNORMAL_ULP = 2.0 ** -149


def rel_err(gpu, ref) -> float:
    """max|gpu - ref| / max|ref| for one output tensor.

    Every output is fp32.  A reference whose whole scale lies below fp32's
    normal range (2^-126), e.g. a gradient that decayed through ~1000 forget
    gates to 1e-189, is checked against its own fp32 rounding instead: each
    GPU value must equal the reference rounded to fp32 (zero or a subnormal)
    within one subnormal ulp (2^-149).  That holds -> 0.0, else inf."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    if ref.size == 0:
        return 0.0
    m = float(np.max(np.abs(ref)))
    if m < FLT_MIN_NORMAL:
        ref32 = ref.astype(np.float32).astype(np.float64)
        return 0.0 if float(np.max(np.abs(gpu - ref32))) <= FLT_SUBNORMAL_ULP else float("inf")
    return float(np.max(np.abs(gpu - ref))) / m


def to_dev(inputs, device, drop=()):
    return {k: (None if k in drop else v.to(device)) for k, v in inputs.items()}


def run_gpu(inputs, device, drop=(), stream=None, mask=None, reverse=False, ijfo=False):
    """Forward + backward through the C ABI.  Inputs named in `drop` are passed
    as NULL (the library treats them as zeros); `mask` (variable length,
    [T,B,H] in the compute type), `reverse` and `ijfo` (gate_order "ijfo")
    select the _ex entry points."""
    order = "ijfo" if ijfo else "ifjo"
    lbuild.build()
    d = to_dev(inputs, device, drop)
    mk = mask.to(device) if mask is not None else None
    s = stream if stream is not None else torch.cuda.current_stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        st = L.forward(d["x"], d["W"], d["b"], d["h0"], d["c0"], stream=s, mask=mk,
                       reverse=reverse, gate_order=order)
        g = L.backward(st, d["x"], d["W"], d["h0"], d["c0"], d["dy"], d["dhT"], d["dcT"],
                       stream=s, mask=mk, reverse=reverse, gate_order=order)
    torch.cuda.synchronize()
    out = dict(y=st.y, hT=st.hT, cT=st.cT, gates=st.gates, cells=st.cells, dx=g.dx, dW=g.dW,
               db=g.db, dh0=g.dh0, dc0=g.dc0)
    return {k: v.float().cpu().double().numpy() for k, v in out.items()}


def run_oracle(inputs, drop=(), mask=None, reverse=False, ijfo=False):
    p = synth.as_float64(inputs)
    for k in drop:
        p[k] = None
    mk = mask.double().numpy() if mask is not None else None
    return oracle.lstm_fwd_bwd(p["x"], p["W"], p["b"], p["h0"], p["c0"], p["dy"], p["dhT"],
                               p["dcT"], mask=mk, reverse=reverse, ijfo=ijfo)


def compare(gpu, ref, dtype, names=OUTS, idx=None):
    """Return {name: rel_err}; `idx` selects the sampled sequences of the GPU
    result (the oracle ran on that sub-batch)."""
    errs = {}
    for k in names:
        g = gpu[k]
        if idx is not None:
            if k in ("y", "dx", "gates", "cells"):
                g = g[:, idx]
            elif k in ("hT", "cT", "dh0", "dc0"):
                g = g[idx]
        errs[k] = rel_err(g, ref[k])
    return errs


def assert_within(errs, dtype, label=""):
    tol = TOL[dtype]
    bad = {k: v for k, v in errs.items() if not (v <= tol)}
    assert not bad, f"{label}: tolerance {tol} exceeded: {bad} (all: {errs})"


def mask_upstream(inputs, idx):
    """Zero dy / dhT / dcT outside the sequences `idx`.  Sequences with no
    upstream gradient contribute exactly zero to dW and db, so the GPU's dW/db
    of the masked problem equals the oracle's dW/db on the sub-batch `idx`."""
    keep = torch.zeros(inputs["x"].shape[1], dtype=torch.bool)
    keep[list(idx)] = True
    out = dict(inputs)
    out["dy"] = torch.where(keep[None, :, None], inputs["dy"], torch.zeros_like(inputs["dy"]))
    out["dhT"] = torch.where(keep[:, None], inputs["dhT"], torch.zeros_like(inputs["dhT"]))
    out["dcT"] = torch.where(keep[:, None], inputs["dcT"], torch.zeros_like(inputs["dcT"]))
    return out
