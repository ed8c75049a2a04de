"""fp64 CPU oracle for the single-layer LSTM forward pass and BPTT.

TEST INFRASTRUCTURE ONLY.  ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` are the only
callers.  The product library never imports this package, and this package
imports nothing from the product library.

The arithmetic lives in ``lstm_oracle.c`` (plain C, fp64, OpenMP over the batch
of independent sequences), which states the forward-formula table and the
"backward algorithm (time step t -> t-1)" of the "SingleLayerLstmGrad" operator
page.  This module only builds that file, marshals numpy arrays into it and
hands the results back.  The stacked (multi-layer) LSTM is the composition of
single-layer calls, written out in ``lstm_stack_fwd`` / ``lstm_stack_bwd``.

Layouts: x[T,B,I], W[4H,H+I] (columns [h | x], rows [i|f|g|o]), b[4H],
h0/c0/hT/cT/dhT/dcT/dh0/dc0 [B,H], y/cells/dy [T,B,H], gates/dG [T,B,4H],
dx [T,B,I], dW [4H,H+I], db [4H].  Every array is float64, C-contiguous.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lstm_oracle.c")
_OUT_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_OUT_DIR, "liblstm_oracle.so")
_lib = None


def compile_source(src: str, out: str) -> str:
    """gcc -O2 -fopenmp: one C file -> one shared library."""
    os.makedirs(os.path.dirname(out), exist_ok=True)
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
           "-Wall", "-Wextra", "-o", tmp, src, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile lstm_oracle.c into oracle/_build/liblstm_oracle.so (gcc, OpenMP)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    return compile_source(_SRC, _LIB_PATH)


def _bind(path: str):
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    i = ctypes.c_int
    lib.oracle_lstm_fwd.argtypes = [i, i, i, i] + [dp] * 5 + [dp] * 5
    lib.oracle_lstm_fwd.restype = i
    lib.oracle_lstm_bwd.argtypes = [i, i, i, i] + [dp] * 9 + [dp] * 6
    lib.oracle_lstm_bwd.restype = i
    lib.oracle_lstm_fwd_ex.argtypes = [i, i, i, i] + [dp] * 6 + [i, i] + [dp] * 5
    lib.oracle_lstm_fwd_ex.restype = i
    lib.oracle_lstm_bwd_ex.argtypes = [i, i, i, i] + [dp] * 5 + [i, i] + [dp] * 5 + [dp] * 6
    lib.oracle_lstm_bwd_ex.restype = i
    lib.oracle_set_threads.argtypes = [i]
    lib.oracle_set_threads.restype = None
    lib.oracle_max_threads.argtypes = []
    lib.oracle_max_threads.restype = i
    return lib


def _load(lib=None):
    global _lib
    if lib is not None:
        return lib
    if _lib is None:
        _lib = _bind(build())
    return _lib


def load_variant(path: str):
    """Bind another build of the oracle source (used by the mutation tests, which
    compile deliberately broken copies to show that the pins catch them)."""
    return _bind(path)


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def _f64(a, shape=None):
    if a is None:
        return None
    if hasattr(a, "detach"):  # torch tensor -> numpy (plain conversion)
        a = a.detach().cpu().double().numpy()
    a = np.ascontiguousarray(a, dtype=np.float64)
    if shape is not None and a.shape != tuple(shape):
        a = a.reshape(shape)
    return a


def _ptr(a):
    if a is None:
        return ctypes.POINTER(ctypes.c_double)()
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def lstm_fwd(x, W, b=None, h0=None, c0=None, lib=None, mask=None, reverse=False, ijfo=False):
    """Forward pass.  Returns dict(y, gates, cells, hT, cT) of float64 arrays.
    mask [T][B][H] (1 = real step, 0 = padding) or None; reverse: the
    recurrence runs over t = T-1 .. 0 (direction "REDIRECTIONAL"); ijfo: gate
    row blocks in the order i, j (= g), f, o (gate_order "ijfo")."""
    x = _f64(x)
    T, B, I = x.shape
    W = _f64(W)
    H = W.shape[0] // 4
    assert W.shape == (4 * H, H + I), (W.shape, H, I)
    b = _f64(b, (4 * H,))
    h0 = _f64(h0, (B, H))
    c0 = _f64(c0, (B, H))
    y = np.empty((T, B, H))
    gates = np.empty((T, B, 4 * H))
    cells = np.empty((T, B, H))
    hT = np.empty((B, H))
    cT = np.empty((B, H))
    mask = _f64(mask, (T, B, H))
    rc = _load(lib).oracle_lstm_fwd_ex(T, B, I, H, _ptr(x), _ptr(W), _ptr(b), _ptr(h0),
                                    _ptr(c0), _ptr(mask), int(bool(reverse)), int(bool(ijfo)),
                                    _ptr(y),
                                    _ptr(gates), _ptr(cells), _ptr(hT), _ptr(cT))
    if rc != 0:
        raise RuntimeError("oracle_lstm_fwd failed")
    return dict(y=y, gates=gates, cells=cells, hT=hT, cT=cT)


def lstm_bwd(x, W, h0, c0, fwd, dy=None, dhT=None, dcT=None, lib=None, mask=None,
             reverse=False, ijfo=False):
    """BPTT given the forward's saved state ``fwd`` (the dict lstm_fwd returns,
    run with the same mask and direction).

    Returns dict(dx, dW, db, dh0, dc0, dG) of float64 arrays; dG holds the
    pre-activation gate gradients [di|df|dg|do] of every step."""
    x = _f64(x)
    T, B, I = x.shape
    W = _f64(W)
    H = W.shape[0] // 4
    h0 = _f64(h0, (B, H))
    c0 = _f64(c0, (B, H))
    dy = _f64(dy, (T, B, H))
    dhT = _f64(dhT, (B, H))
    dcT = _f64(dcT, (B, H))
    y, gates, cells = (_f64(fwd[k]) for k in ("y", "gates", "cells"))
    dx = np.empty((T, B, I))
    dW = np.empty((4 * H, H + I))
    db = np.empty((4 * H,))
    dh0 = np.empty((B, H))
    dc0 = np.empty((B, H))
    dG = np.empty((T, B, 4 * H))
    mask = _f64(mask, (T, B, H))
    rc = _load(lib).oracle_lstm_bwd_ex(T, B, I, H, _ptr(x), _ptr(W), _ptr(h0), _ptr(c0),
                                    _ptr(mask), int(bool(reverse)), int(bool(ijfo)), _ptr(y),
                                    _ptr(gates),
                                    _ptr(cells),
                                 _ptr(dy), _ptr(dhT), _ptr(dcT),
                                 _ptr(dx), _ptr(dW), _ptr(db), _ptr(dh0), _ptr(dc0), _ptr(dG))
    if rc != 0:
        raise RuntimeError("oracle_lstm_bwd failed")
    return dict(dx=dx, dW=dW, db=db, dh0=dh0, dc0=dc0, dG=dG)


def lstm_fwd_bwd(x, W, b=None, h0=None, c0=None, dy=None, dhT=None, dcT=None, lib=None,
                 mask=None, reverse=False, ijfo=False):
    """Forward then backward; returns the union of both result dicts."""
    f = lstm_fwd(x, W, b, h0, c0, lib=lib, mask=mask, reverse=reverse, ijfo=ijfo)
    g = lstm_bwd(x, W, h0, c0, f, dy, dhT, dcT, lib=lib, mask=mask, reverse=reverse, ijfo=ijfo)
    out = dict(f)
    out.update(g)
    return out


def lstm_stack_fwd(x, Ws, bs=None, h0s=None, c0s=None, lib=None, mask=None, reverse=False,
                   ijfo=False):
    """Stacked LSTM forward ("cmu 10-414 HW4" page, the multi-layer LSTM
    module's forward; "mxnet-lstm" page, "Stack Multiple RNN Cells"): layer 0
    runs the single-layer cell on x; layer l > 0 runs it on the outputs y of
    layer l-1.  Layer l has its own W_l [4H, H + I_l] (I_0 = I, I_l = H after),
    b_l and initial state h0s[l], c0s[l] [B, H]; its final state is kept apart
    (hT / cT per layer) and only y passes upward.  mask / reverse / ijfo apply
    to every layer.  Returns the list of per-layer forward dicts; the stack's
    output is the last one's "y"."""
    L = len(Ws)
    out, inp = [], x
    for l in range(L):
        f = lstm_fwd(inp, Ws[l], None if bs is None else bs[l],
                     None if h0s is None else h0s[l], None if c0s is None else c0s[l],
                     lib=lib, mask=mask, reverse=reverse, ijfo=ijfo)
        out.append(f)
        inp = f["y"]
    return out


def lstm_stack_bwd(x, Ws, h0s, c0s, fwds, dy=None, dhTs=None, dcTs=None, lib=None, mask=None,
                   reverse=False, ijfo=False):
    """Stacked LSTM backward: the chain rule through the composition of
    lstm_stack_fwd.  The top layer takes dy; layer l-1 takes the gradient at
    its outputs y, which is the dx of layer l; dhTs[l] / dcTs[l] enter at layer
    l's final state.  Returns the list of per-layer gradient dicts (layer 0's
    "dx" is the gradient at x)."""
    L = len(Ws)
    grads = [None] * L
    up = dy
    for l in reversed(range(L)):
        xin = x if l == 0 else fwds[l - 1]["y"]
        g = lstm_bwd(xin, Ws[l], None if h0s is None else h0s[l],
                     None if c0s is None else c0s[l], fwds[l], up,
                     None if dhTs is None else dhTs[l], None if dcTs is None else dcTs[l],
                     lib=lib, mask=mask, reverse=reverse, ijfo=ijfo)
        grads[l] = g
        up = g["dx"]
    return grads


def surrogate_loss(fwd, dy=None, dhT=None, dcT=None) -> float:
    """L = sum_t <dy_t, h_t> + <dhT, h_{T-1}> + <dcT, c_{T-1}>: the scalar whose
    gradient the dy / dh / dc inputs of the backward pass define."""
    L = 0.0
    if dy is not None:
        L += float(np.sum(_f64(dy) * fwd["y"]))
    if dhT is not None:
        L += float(np.sum(_f64(dhT) * fwd["hT"]))
    if dcT is not None:
        L += float(np.sum(_f64(dcT) * fwd["cT"]))
    return L
