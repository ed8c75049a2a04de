"""Pins for the fp64 oracle, independent of the oracle's own backward formulas.

Every gradient the oracle returns is checked against something other than
itself: central finite differences of the surrogate loss, complex-step
derivatives of a hand-written scalar forward, torch.nn.LSTM with autograd in
fp64, and closed forms that follow from the chain rule in special cases.
Formulas come from the "SingleLayerLstmGrad" operator page (forward-formula
table, backward algorithm steps 1-6, gradient derivation, parameter table) and
the test recipes of the DarkNetLSTMLayer page (hand example with zero and
non-zero initial state, finite differences, batch vs step-by-step forward).
"""
import cmath
import math

import numpy as np
import pytest
import torch

import oracle
from backward_lstm_fwd_b200 import synth

GRAD_OF = {"x": "dx", "W": "dW", "b": "db", "h0": "dh0", "c0": "dc0"}


def random_case(T, B, I, H, seed, wscale=1.5, dhdc=True, dy=True):
    r = np.random.default_rng(seed)
    p = dict(
        x=r.uniform(-1, 1, (T, B, I)),
        W=r.uniform(-1, 1, (4 * H, H + I)) * wscale / math.sqrt(max(H, 1)),
        b=r.uniform(-1, 1, (4 * H,)) * 0.5,
        h0=r.normal(0, 0.5, (B, H)),
        c0=r.normal(0, 0.5, (B, H)),
    )
    g = dict(
        dy=r.normal(0, 1, (T, B, H)) if dy else np.zeros((T, B, H)),
        dhT=r.normal(0, 1, (B, H)) if dhdc else np.zeros((B, H)),
        dcT=r.normal(0, 1, (B, H)) if dhdc else np.zeros((B, H)),
    )
    return p, g


def run(p, g, lib=None, mask=None, reverse=False, ijfo=False):
    return oracle.lstm_fwd_bwd(p["x"], p["W"], p["b"], p["h0"], p["c0"],
                               g["dy"], g["dhT"], g["dcT"], lib=lib, mask=mask, reverse=reverse,
                               ijfo=ijfo)


def loss(p, g, lib=None, mask=None, reverse=False, ijfo=False):
    f = oracle.lstm_fwd(p["x"], p["W"], p["b"], p["h0"], p["c0"], lib=lib, mask=mask,
                        reverse=reverse, ijfo=ijfo)
    return oracle.surrogate_loss(f, g["dy"], g["dhT"], g["dcT"])


def fd_max_error(p, g, lib=None, max_entries=None, seed=0, mask=None, reverse=False,
                 ijfo=False):
    """max over checked entries of |analytic - central FD| / max(1, |analytic|)."""
    out = run(p, g, lib, mask, reverse, ijfo)
    rng = np.random.default_rng(seed)
    worst = 0.0
    for name, gname in GRAD_OF.items():
        theta = p[name]
        an = out[gname].reshape(-1)
        idx = np.arange(theta.size)
        if max_entries is not None and theta.size > max_entries:
            idx = rng.choice(theta.size, max_entries, replace=False)
        flat = theta.reshape(-1)
        for k in idx:
            old = flat[k]
            h = 1e-6 * max(1.0, abs(old))
            flat[k] = old + h
            lp = loss(p, g, lib, mask, reverse, ijfo)
            flat[k] = old - h
            lm = loss(p, g, lib, mask, reverse, ijfo)
            flat[k] = old
            fd = (lp - lm) / (2 * h)
            worst = max(worst, abs(fd - an[k]) / max(1.0, abs(an[k])))
    return worst


@pytest.mark.parametrize("T,B,I,H,dhdc", [
    (1, 2, 3, 4, True), (2, 2, 3, 4, True), (3, 2, 3, 4, True),
    (3, 1, 2, 5, False), (2, 3, 1, 2, True), (3, 2, 4, 3, True),
])
def test_finite_differences_small(T, B, I, H, dhdc):
    p, g = random_case(T, B, I, H, seed=10 * T + H, dhdc=dhdc)
    assert fd_max_error(p, g) < 1e-6


def test_finite_differences_tiny_workload():
    """The 8-step, batch-2, I=16, H=32 fp32 workload's own inputs."""
    w = synth.WORKLOADS["lstm_T8_B2_I16_H32_fp32"]
    inp = synth.as_float64(synth.make_inputs(w))
    p = {k: inp[k].copy() for k in ("x", "W", "b", "h0", "c0")}
    g = {k: inp[k] for k in ("dy", "dhT", "dcT")}
    # the workload has dhT = dcT = 0; also check with them drawn
    assert fd_max_error(p, g, max_entries=400) < 1e-6
    r = np.random.default_rng(5)
    g2 = dict(g, dhT=r.normal(size=g["dhT"].shape), dcT=r.normal(size=g["dcT"].shape))
    assert fd_max_error(p, g2, max_entries=200, seed=1) < 1e-6


def test_against_torch_lstm_fp64():
    """torch.nn.LSTM (gate rows i, f, g, o; weight_ih = W_x, weight_hh = W_h,
    bias_ih = b, bias_hh = 0) with autograd, all in fp64 on the CPU."""
    T, B, I, H = 5, 3, 6, 7
    p, g = random_case(T, B, I, H, seed=3)
    out = run(p, g)

    lstm = torch.nn.LSTM(I, H).double()
    with torch.no_grad():
        lstm.weight_ih_l0.copy_(torch.from_numpy(p["W"][:, H:]))
        lstm.weight_hh_l0.copy_(torch.from_numpy(p["W"][:, :H]))
        lstm.bias_ih_l0.copy_(torch.from_numpy(p["b"]))
        lstm.bias_hh_l0.zero_()
    x = torch.from_numpy(p["x"]).requires_grad_()
    h0 = torch.from_numpy(p["h0"])[None].clone().requires_grad_()
    c0 = torch.from_numpy(p["c0"])[None].clone().requires_grad_()
    y, (hn, cn) = lstm(x, (h0, c0))
    L = ((torch.from_numpy(g["dy"]) * y).sum() + (torch.from_numpy(g["dhT"]) * hn[0]).sum()
         + (torch.from_numpy(g["dcT"]) * cn[0]).sum())
    L.backward()
    dW = torch.cat([lstm.weight_hh_l0.grad, lstm.weight_ih_l0.grad], dim=1)

    def close(a, b):
        np.testing.assert_allclose(a, b.detach().numpy(), rtol=1e-10, atol=1e-12)

    close(out["y"], y)
    close(out["hT"], hn[0])
    close(out["cT"], cn[0])
    close(out["dx"], x.grad)
    close(out["dW"], dW)
    close(out["db"], lstm.bias_ih_l0.grad)
    close(out["dh0"], h0.grad[0])
    close(out["dc0"], c0.grad[0])


def _scalar_forward(theta, x, h0, c0):
    """H = I = B = 1 forward written from the forward-formula table with complex
    arithmetic, so that complex-step derivatives are exact to rounding.
    theta = [W_ih, W_ix, W_fh, W_fx, W_gh, W_gx, W_oh, W_ox, b_i, b_f, b_g, b_o]."""
    sig = lambda a: 1.0 / (1.0 + cmath.exp(-a))
    h, c = h0, c0
    hs, cs = [], []
    for xt in x:
        i = sig(theta[0] * h + theta[1] * xt + theta[8])
        f = sig(theta[2] * h + theta[3] * xt + theta[9])
        g = cmath.tanh(theta[4] * h + theta[5] * xt + theta[10])
        o = sig(theta[6] * h + theta[7] * xt + theta[11])
        c = f * c + i * g
        h = o * cmath.tanh(c)
        hs.append(h)
        cs.append(c)
    return hs, cs


@pytest.mark.parametrize("h0,c0", [(0.0, 0.0), (0.7, -1.3)])
def test_hand_example_two_steps(h0, c0):
    """Hidden, input and batch size 1, two steps (DarkNetLSTMLayer page test recipe),
    once with zero and once with non-zero initial state; gradients by complex step."""
    theta = [0.5, -0.25, 0.75, 0.125, -0.5, 1.0, 0.25, -0.75, 0.1, -0.2, 0.3, 0.05]
    xs = [1.0, -0.5]
    dy = [0.3, -1.1]
    dhT, dcT = 0.4, -0.6

    def L(th, x, hh, cc):
        hs, cs = _scalar_forward(th, x, hh, cc)
        return sum(d * h for d, h in zip(dy, hs)) + dhT * hs[-1] + dcT * cs[-1]

    hs, cs = _scalar_forward(theta, xs, h0, c0)
    W = np.array([[theta[0], theta[1]], [theta[2], theta[3]],
                  [theta[4], theta[5]], [theta[6], theta[7]]])
    b = np.array(theta[8:12])
    out = oracle.lstm_fwd_bwd(np.array(xs).reshape(2, 1, 1), W, b, np.array([[h0]]),
                              np.array([[c0]]), np.array(dy).reshape(2, 1, 1),
                              np.array([[dhT]]), np.array([[dcT]]))
    np.testing.assert_allclose(out["y"].ravel(), [h.real for h in hs], rtol=1e-14)
    np.testing.assert_allclose(out["cells"].ravel(), [c.real for c in cs], rtol=1e-14)

    eps = 1e-30
    def cstep(fn):
        return fn(eps * 1j).imag / eps
    dW = np.zeros(8)
    for k in range(8):
        dW[k] = cstep(lambda e: L([t + (e if j == k else 0) for j, t in enumerate(theta)], xs, h0, c0))
    db = np.array([cstep(lambda e: L([t + (e if j == 8 + k else 0) for j, t in enumerate(theta)],
                                     xs, h0, c0)) for k in range(4)])
    dx = np.array([cstep(lambda e: L(theta, [v + (e if j == k else 0) for j, v in enumerate(xs)],
                                     h0, c0)) for k in range(2)])
    dh0 = cstep(lambda e: L(theta, xs, h0 + e, c0))
    dc0 = cstep(lambda e: L(theta, xs, h0, c0 + e))
    np.testing.assert_allclose(out["dW"].ravel(), dW, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(out["db"], db, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(out["dx"].ravel(), dx, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(out["dh0"].ravel(), [dh0], rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(out["dc0"].ravel(), [dc0], rtol=1e-12, atol=1e-15)


def test_zero_weights_closed_form():
    """W = 0, b = 0: every gate pre-activation is 0, so i = f = o = 1/2, g = 0,
    c_t = c0 / 2^(t+1), h_t = tanh(c_t) / 2.  h no longer feeds back, so
    dL/dc_t = sum_{s >= t} 2^-(s-t) e_s with e_s = dh_s * (1 - tanh^2 c_s) / 2
    (+ dcT at s = T-1) and dh_s = dy_s (+ dhT at s = T-1), from the chain rule
    (product of forget gates, gradient derivation section)."""
    T, B, I, H = 6, 3, 4, 5
    r = np.random.default_rng(7)
    x = r.uniform(-1, 1, (T, B, I))
    W = np.zeros((4 * H, H + I))
    b = np.zeros(4 * H)
    h0, c0 = r.normal(0, 1, (B, H)), r.normal(0, 1, (B, H))
    dy, dhT, dcT = r.normal(size=(T, B, H)), r.normal(size=(B, H)), r.normal(size=(B, H))
    out = oracle.lstm_fwd_bwd(x, W, b, h0, c0, dy, dhT, dcT)

    c = np.stack([c0 / 2.0 ** (t + 1) for t in range(T)])
    h = 0.5 * np.tanh(c)
    np.testing.assert_allclose(out["cells"], c, rtol=1e-15)
    np.testing.assert_allclose(out["y"], h, rtol=1e-15)
    np.testing.assert_allclose(out["gates"][..., :2 * H], 0.5)
    np.testing.assert_allclose(out["gates"][..., 2 * H:3 * H], 0.0)
    np.testing.assert_allclose(out["gates"][..., 3 * H:], 0.5)

    dh = dy.copy()
    dh[-1] += dhT
    e = dh * 0.5 * (1 - np.tanh(c) ** 2)
    e[-1] += dcT
    dc = np.stack([sum(e[s] * 0.5 ** (s - t) for s in range(t, T)) for t in range(T)])
    cprev = np.concatenate([c0[None], c[:-1]])
    d_i = np.zeros_like(dc)                       # g = 0
    d_f = dc * cprev * 0.25
    d_g = dc * 0.5
    d_o = dh * np.tanh(c) * 0.25
    dG = np.concatenate([d_i, d_f, d_g, d_o], axis=-1)
    hprev = np.concatenate([h0[None], h[:-1]])
    z = np.concatenate([hprev, x], axis=-1)
    np.testing.assert_allclose(out["dG"], dG, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(out["dW"], np.einsum("tbr,tbk->rk", dG, z), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(out["db"], dG.sum((0, 1)), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(out["dx"], 0.0)
    np.testing.assert_allclose(out["dh0"], 0.0)
    np.testing.assert_allclose(out["dc0"], 0.5 * dc[0], rtol=1e-12, atol=1e-14)


def test_one_step_closed_form():
    """T = 1 in closed form: with z = W [h0; x_0] + b, i, f, o = sigma(z_i, z_f,
    z_o), g = tanh(z_g), the forward table gives c = f c0 + i g and y_0 = hT =
    o tanh(c).  That expression, written out in torch (fp64) and differentiated
    by autograd, gives every gradient of L = <dy_0 + dhT, h> + <dcT, c>."""
    B, I, H = 3, 4, 5
    p, g = random_case(1, B, I, H, seed=21)
    out = run(p, g)
    t = {k: torch.from_numpy(np.array(v)).requires_grad_() for k, v in p.items()}
    z = torch.cat([t["h0"], t["x"][0]], dim=1) @ t["W"].T + t["b"]
    i, f = torch.sigmoid(z[:, :H]), torch.sigmoid(z[:, H:2 * H])
    gg, o = torch.tanh(z[:, 2 * H:3 * H]), torch.sigmoid(z[:, 3 * H:])
    c = f * t["c0"] + i * gg
    h = o * torch.tanh(c)
    L = ((torch.from_numpy(g["dy"][0]) + torch.from_numpy(g["dhT"])) * h).sum() + \
        (torch.from_numpy(g["dcT"]) * c).sum()
    L.backward()

    def close(a, b):
        np.testing.assert_allclose(a, b.detach().numpy(), rtol=1e-12, atol=1e-14)

    close(out["y"][0], h)
    close(out["hT"], h)
    close(out["cT"], c)
    close(out["dx"], t["x"].grad)
    close(out["dW"], t["W"].grad)
    close(out["db"], t["b"].grad)
    close(out["dh0"], t["h0"].grad)
    close(out["dc0"], t["c0"].grad)


def test_invariants():
    """db = sum over t and batch of dG; dW = sum dG z^T; dx_t and dh_prev are the
    x- and h-parts of W^T dG_t; delta c_prev = delta c_t * f_t (steps 4-5)."""
    T, B, I, H = 4, 3, 5, 6
    p, g = random_case(T, B, I, H, seed=11, wscale=1.0)
    out = run(p, g)
    dG, W = out["dG"], p["W"]
    np.testing.assert_allclose(out["db"], dG.sum((0, 1)), rtol=1e-12, atol=1e-13)
    hprev = np.concatenate([p["h0"][None], out["y"][:-1]])
    z = np.concatenate([hprev, p["x"]], axis=-1)
    np.testing.assert_allclose(out["dW"], np.einsum("tbr,tbk->rk", dG, z), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(out["dx"], dG @ W[:, H:], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(out["dh0"], dG[0] @ W[:, :H], rtol=1e-12, atol=1e-13)
    i0, f0, g0 = (out["gates"][0][:, k * H:(k + 1) * H] for k in range(3))
    dc_0 = dG[0][:, 2 * H:3 * H] / (i0 * (1 - g0 ** 2))   # dg = dc * i * (1 - g^2)
    np.testing.assert_allclose(out["dc0"], dc_0 * f0, rtol=1e-9, atol=1e-12)


def test_linearity_in_upstream_gradients():
    p, g = random_case(3, 2, 3, 4, seed=21)
    a = run(p, g)
    alpha = -2.5
    b = run(p, {k: alpha * v for k, v in g.items()})
    for k in ("dx", "dW", "db", "dh0", "dc0"):
        np.testing.assert_allclose(b[k], alpha * a[k], rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("split", [1, 3, 5])
def test_chunked_equals_whole(split):
    """A T-step call equals two chained calls (DarkNetLSTMLayer page: batch vs
    step-by-step forward).  Backward chains through dh/dc: the second chunk's
    d initH / d initC are the first chunk's dh / dc inputs."""
    T, B, I, H = 6, 2, 3, 4
    p, g = random_case(T, B, I, H, seed=31)
    whole = run(p, g)
    p1 = dict(p, x=p["x"][:split])
    p2 = dict(p, x=p["x"][split:], h0=whole["y"][split - 1], c0=whole["cells"][split - 1])
    g2 = dict(g, dy=g["dy"][split:])
    second = run(p2, g2)
    first = run(p1, dict(dy=g["dy"][:split], dhT=second["dh0"], dcT=second["dc0"]))
    np.testing.assert_allclose(np.concatenate([first["y"], second["y"]]), whole["y"], rtol=1e-14)
    np.testing.assert_allclose(second["hT"], whole["hT"], rtol=1e-14)
    np.testing.assert_allclose(second["cT"], whole["cT"], rtol=1e-14)
    np.testing.assert_allclose(np.concatenate([first["dx"], second["dx"]]), whole["dx"],
                               rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(first["dW"] + second["dW"], whole["dW"], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(first["db"] + second["db"], whole["db"], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(first["dh0"], whole["dh0"], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(first["dc0"], whole["dc0"], rtol=1e-12, atol=1e-14)


def test_batch_rows_are_independent():
    p, g = random_case(4, 5, 3, 4, seed=41)
    whole = run(p, g)
    idx = [3, 1]
    sub = run(dict(p, x=p["x"][:, idx], h0=p["h0"][idx], c0=p["c0"][idx]),
              dict(dy=g["dy"][:, idx], dhT=g["dhT"][idx], dcT=g["dcT"][idx]))
    np.testing.assert_allclose(sub["y"], whole["y"][:, idx], rtol=1e-14)
    np.testing.assert_allclose(sub["dx"], whole["dx"][:, idx], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(sub["dh0"], whole["dh0"][idx], rtol=1e-12, atol=1e-14)


def test_empty_sequence_and_batch():
    p, g = random_case(0, 2, 3, 4, seed=1)
    out = run(p, g)
    np.testing.assert_array_equal(out["hT"], p["h0"])
    np.testing.assert_array_equal(out["cT"], p["c0"])
    np.testing.assert_array_equal(out["dh0"], g["dhT"])
    np.testing.assert_array_equal(out["dc0"], g["dcT"])
    np.testing.assert_array_equal(out["dW"], 0.0)
    np.testing.assert_array_equal(out["db"], 0.0)
    p, g = random_case(3, 0, 3, 4, seed=1)
    out = run(p, g)
    assert out["y"].shape == (3, 0, 4)
    np.testing.assert_array_equal(out["dW"], 0.0)


# ---------------------------------------------------------------- seq_length
# The parameter table's optional "seq_length" mask [T][B][H], read as 1 = real
# step, 0 = padding: padding keeps the state (c_t = c_{t-1}, h_t = h_{t-1}) and
# passes delta h / delta c through (the Darknet LSTM page's note that padding
# must not update state or gradients).

def random_mask(T, B, H, seed, p_pad=0.35):
    return (np.random.default_rng(seed).random((T, B, H)) >= p_pad).astype(np.float64)


@pytest.mark.parametrize("T,B,I,H", [(3, 2, 3, 4), (4, 3, 2, 5), (2, 1, 3, 3)])
def test_masked_finite_differences(T, B, I, H):
    """The masked backward is the gradient of the masked forward (0/1 mask per
    element, fixed while differentiating)."""
    p, g = random_case(T, B, I, H, seed=300 + T * H)
    mask = random_mask(T, B, H, seed=7 + T)
    assert fd_max_error(p, g, mask=mask) < 1e-6


def test_mask_all_ones_is_unmasked():
    p, g = random_case(4, 3, 5, 6, seed=41)
    a = run(p, g)
    b = run(p, g, mask=np.ones((4, 3, 6)))
    for k in a:
        np.testing.assert_array_equal(a[k], b[k], err_msg=k)


def test_length_mask_equals_truncated_sequences():
    """With mask[t, n, :] = (t < L_n) every sequence behaves as the unmasked
    LSTM run on its first L_n steps: outputs and gradients on those steps agree,
    padded steps carry the final state and get no input gradient, the dy of
    padded steps reaches h_{L_n - 1} (its value is carried there), and dW / db
    are the sums over the truncated runs.  Lengths include 0 and T."""
    T, B, I, H = 6, 5, 3, 4
    p, g = random_case(T, B, I, H, seed=77)
    lengths = [6, 0, 3, 1, 5]
    mask = np.zeros((T, B, H))
    for n, L in enumerate(lengths):
        mask[:L, n, :] = 1.0
    out = run(p, g, mask=mask)
    dW = np.zeros_like(out["dW"])
    db = np.zeros_like(out["db"])
    for n, L in enumerate(lengths):
        sl = slice(n, n + 1)
        q = dict(x=p["x"][:L, sl], W=p["W"], b=p["b"], h0=p["h0"][sl], c0=p["c0"][sl])
        dhT = g["dhT"][sl] + g["dy"][L:, sl].sum(axis=0)
        ref = run(q, dict(dy=g["dy"][:L, sl], dhT=dhT, dcT=g["dcT"][sl]))
        close = lambda a, b: np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)
        close(out["y"][:L, sl], ref["y"])
        close(out["gates"][:L, sl], ref["gates"])
        close(out["cells"][:L, sl], ref["cells"])
        close(out["hT"][sl], ref["hT"])
        close(out["cT"][sl], ref["cT"])
        for t in range(L, T):  # padding carries the final state
            close(out["y"][t, sl], ref["hT"])
            close(out["cells"][t, sl], ref["cT"])
        close(out["dx"][:L, sl], ref["dx"])
        assert not out["dx"][L:, sl].any()
        close(out["dh0"][sl], ref["dh0"])
        close(out["dc0"][sl], ref["dc0"])
        dW += ref["dW"]
        db += ref["db"]
    np.testing.assert_allclose(out["dW"], dW, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(out["db"], db, rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------- direction
# The operator's "direction" attribute: "REDIRECTIONAL" runs the recurrence over
# t = T-1 .. 0 (initH / initC before step t = T-1; hT / cT after step t = 0).

@pytest.mark.parametrize("T,B,I,H,masked", [(3, 2, 3, 4, False), (4, 2, 2, 3, True)])
def test_reverse_finite_differences(T, B, I, H, masked):
    p, g = random_case(T, B, I, H, seed=500 + T * H)
    mask = random_mask(T, B, H, seed=9 + T) if masked else None
    assert fd_max_error(p, g, mask=mask, reverse=True) < 1e-6


def test_reverse_is_forward_on_flipped_time():
    """The reverse LSTM is the forward LSTM on the time-flipped sequences, its
    per-step outputs flipped back: y, gates, cells, dx (and the mask) flip;
    hT, cT, dW, db, dh0, dc0 are the same."""
    T, B, I, H = 5, 3, 4, 6
    p, g = random_case(T, B, I, H, seed=91)
    mask = random_mask(T, B, H, seed=92)
    rev = run(p, g, mask=mask, reverse=True)
    pf = dict(p, x=p["x"][::-1].copy())
    gf = dict(g, dy=g["dy"][::-1].copy())
    fwd = run(pf, gf, mask=mask[::-1].copy())
    for k in ("y", "gates", "cells", "dx"):
        np.testing.assert_allclose(rev[k], fwd[k][::-1], rtol=1e-12, atol=1e-13, err_msg=k)
    for k in ("hT", "cT", "dW", "db", "dh0", "dc0"):
        np.testing.assert_allclose(rev[k], fwd[k], rtol=1e-11, atol=1e-12, err_msg=k)


# ---------------------------------------------------------------- gate order
# The operator's "gate_order" attribute: "ifjo" (the default reading) or
# "ijfo", the row blocks of W, b, the saved gates and dG in the order i, j, f, o.

def _swap_fg_blocks(a, H, axis):
    """Exchange row blocks 1 and 2 (f and j) of a [.. 4H ..] array."""
    idx = np.r_[0:H, 2 * H:3 * H, H:2 * H, 3 * H:4 * H]
    return np.take(a, idx, axis=axis)


def test_ijfo_finite_differences():
    p, g = random_case(3, 2, 3, 4, seed=611)
    assert fd_max_error(p, g, ijfo=True) < 1e-6


def test_ijfo_is_ifjo_with_blocks_swapped():
    """gate_order "ijfo" on W, b equals "ifjo" on the same weights with row
    blocks 1 and 2 exchanged; gates, dG-shaped outputs (dW rows, db) come back
    with the blocks exchanged, everything else equal."""
    T, B, I, H = 4, 3, 5, 6
    p, g = random_case(T, B, I, H, seed=612)
    a = run(p, g, ijfo=True)
    q = dict(p, W=_swap_fg_blocks(p["W"], H, 0), b=_swap_fg_blocks(p["b"], H, 0))
    r = run(q, g)
    for k in ("y", "cells", "hT", "cT", "dx", "dh0", "dc0"):
        np.testing.assert_allclose(a[k], r[k], rtol=1e-12, atol=1e-13, err_msg=k)
    np.testing.assert_allclose(a["gates"], _swap_fg_blocks(r["gates"], H, 2), rtol=1e-12,
                               atol=1e-13)
    np.testing.assert_allclose(a["dW"], _swap_fg_blocks(r["dW"], H, 0), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(a["db"], _swap_fg_blocks(r["db"], H, 0), rtol=1e-11, atol=1e-12)
