"""Pins for the stacked-LSTM oracle (layer l runs the single-layer cell on
layer l-1's outputs: the multi-layer LSTM module of the "cmu 10-414 HW4" page,
"Stack Multiple RNN Cells" of the "mxnet-lstm" page).  The composition and
its chain rule are checked against torch.nn.LSTM(num_layers=L) with autograd
in fp64, and against central finite differences of the stack's surrogate loss
(also with a mask, the reverse direction and gate_order "ijfo")."""
import math

import numpy as np
import pytest
import torch

import oracle


def stack_case(T, B, I, H, L, seed):
    r = np.random.default_rng(seed)
    p = dict(x=r.uniform(-1, 1, (T, B, I)))
    p["W"] = [r.uniform(-1, 1, (4 * H, H + (I if l == 0 else H))) * 1.5 / math.sqrt(H)
              for l in range(L)]
    p["b"] = [r.uniform(-0.5, 0.5, (4 * H,)) for _ in range(L)]
    p["h0"] = [r.normal(0, 0.5, (B, H)) for _ in range(L)]
    p["c0"] = [r.normal(0, 0.5, (B, H)) for _ in range(L)]
    g = dict(dy=r.normal(0, 1, (T, B, H)),
             dhT=[r.normal(0, 1, (B, H)) for _ in range(L)],
             dcT=[r.normal(0, 1, (B, H)) for _ in range(L)])
    return p, g


def run_stack(p, g, **opt):
    f = oracle.lstm_stack_fwd(p["x"], p["W"], p["b"], p["h0"], p["c0"], **opt)
    gr = oracle.lstm_stack_bwd(p["x"], p["W"], p["h0"], p["c0"], f, g["dy"], g["dhT"], g["dcT"],
                               **opt)
    return f, gr


def stack_loss(p, g, **opt):
    f = oracle.lstm_stack_fwd(p["x"], p["W"], p["b"], p["h0"], p["c0"], **opt)
    L = float(np.sum(g["dy"] * f[-1]["y"]))
    for l, fl in enumerate(f):
        L += float(np.sum(g["dhT"][l] * fl["hT"]) + np.sum(g["dcT"][l] * fl["cT"]))
    return L


@pytest.mark.parametrize("L", [2, 3])
def test_stack_matches_torch_lstm(L):
    T, B, I, H = 5, 3, 6, 4
    p, g = stack_case(T, B, I, H, L, seed=20 + L)
    f, gr = run_stack(p, g)
    lstm = torch.nn.LSTM(I, H, num_layers=L).double()
    with torch.no_grad():
        for l in range(L):
            getattr(lstm, f"weight_ih_l{l}").copy_(torch.from_numpy(p["W"][l][:, H:]))
            getattr(lstm, f"weight_hh_l{l}").copy_(torch.from_numpy(p["W"][l][:, :H]))
            getattr(lstm, f"bias_ih_l{l}").copy_(torch.from_numpy(p["b"][l]))
            getattr(lstm, f"bias_hh_l{l}").zero_()
    x = torch.from_numpy(p["x"]).requires_grad_()
    h0 = torch.from_numpy(np.stack(p["h0"])).requires_grad_()
    c0 = torch.from_numpy(np.stack(p["c0"])).requires_grad_()
    y, (hn, cn) = lstm(x, (h0, c0))
    loss = ((torch.from_numpy(g["dy"]) * y).sum()
            + (torch.from_numpy(np.stack(g["dhT"])) * hn).sum()
            + (torch.from_numpy(np.stack(g["dcT"])) * cn).sum())
    loss.backward()

    def close(a, b):
        np.testing.assert_allclose(a, b.detach().numpy(), rtol=1e-10, atol=1e-12)

    close(f[-1]["y"], y)
    close(gr[0]["dx"], x.grad)
    for l in range(L):
        close(f[l]["hT"], hn[l])
        close(f[l]["cT"], cn[l])
        close(gr[l]["dh0"], h0.grad[l])
        close(gr[l]["dc0"], c0.grad[l])
        dW = torch.cat([getattr(lstm, f"weight_hh_l{l}").grad,
                        getattr(lstm, f"weight_ih_l{l}").grad], dim=1)
        close(gr[l]["dW"], dW)
        close(gr[l]["db"], getattr(lstm, f"bias_ih_l{l}").grad)


def test_one_layer_stack_is_the_single_layer():
    p, g = stack_case(4, 2, 3, 5, 1, seed=9)
    f, gr = run_stack(p, g)
    one = oracle.lstm_fwd_bwd(p["x"], p["W"][0], p["b"][0], p["h0"][0], p["c0"][0], g["dy"],
                              g["dhT"][0], g["dcT"][0])
    for k in ("y", "hT", "cT"):
        np.testing.assert_array_equal(f[0][k], one[k])
    for k in ("dx", "dW", "db", "dh0", "dc0"):
        np.testing.assert_array_equal(gr[0][k], one[k])


@pytest.mark.parametrize("opts", [{}, {"reverse": True, "ijfo": True}, {"masked": True}])
def test_stack_finite_differences(opts):
    T, B, I, H, L = 3, 2, 3, 4, 2
    p, g = stack_case(T, B, I, H, L, seed=31)
    opt = {k: v for k, v in opts.items() if k != "masked"}
    if opts.get("masked"):
        r = np.random.default_rng(5)
        opt["mask"] = (r.uniform(size=(T, B, H)) < 0.7).astype(np.float64)
    f, gr = run_stack(p, g, **opt)
    worst = 0.0
    params = [("x", None, gr[0]["dx"])]
    for l in range(L):
        params += [("W", l, gr[l]["dW"]), ("b", l, gr[l]["db"]), ("h0", l, gr[l]["dh0"]),
                   ("c0", l, gr[l]["dc0"])]
    for name, l, an in params:
        theta = p[name] if l is None else p[name][l]
        flat, an = theta.reshape(-1), an.reshape(-1)
        for k in range(flat.size):
            old = flat[k]
            h = 1e-6 * max(1.0, abs(old))
            flat[k] = old + h
            lp = stack_loss(p, g, **opt)
            flat[k] = old - h
            lm = stack_loss(p, g, **opt)
            flat[k] = old
            worst = max(worst, abs((lp - lm) / (2 * h) - an[k]) / max(1.0, abs(an[k])))
    assert worst < 1e-6
