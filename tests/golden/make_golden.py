"""Write the oracle regression fixtures of tests/golden/.

None of the pages ("SingleLayerLstmGrad", the MXNet, Darknet, PyTorch GRU and
CMU 10-414 pages) prints a worked numerical example, so no stored value here
comes from a page.  These fixtures record what the fp64 oracle returns on a
few small seeded problems -- default options, the reverse direction with a
mask, gate_order "ijfo", and a two-layer stack -- so that any later change to
the oracle's arithmetic shows up as a diff of these files (and must then name
the passage that justifies it).  They are not pins of correctness; the pins
are in tests/test_oracle*.py.

    python tests/golden/make_golden.py      # rewrites the .json files
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402


def case_inputs(T, B, I, H, seed, layers=1):
    r = np.random.default_rng(seed)
    p = {"x": r.uniform(-1, 1, (T, B, I)),
         "W": [r.uniform(-0.6, 0.6, (4 * H, H + (I if l == 0 else H))) for l in range(layers)],
         "b": [r.uniform(-0.3, 0.3, (4 * H,)) for _ in range(layers)],
         "h0": [r.normal(0, 0.5, (B, H)) for _ in range(layers)],
         "c0": [r.normal(0, 0.5, (B, H)) for _ in range(layers)],
         "dy": r.normal(0, 1, (T, B, H)),
         "dhT": [r.normal(0, 1, (B, H)) for _ in range(layers)],
         "dcT": [r.normal(0, 1, (B, H)) for _ in range(layers)]}
    return p


CASES = {
    "lstm_T3_B2_I3_H4_ifjo": dict(T=3, B=2, I=3, H=4, seed=7),
    "lstm_T3_B2_I3_H4_reverse_mask": dict(T=3, B=2, I=3, H=4, seed=8, reverse=True, mask=True),
    "lstm_T3_B2_I3_H4_ijfo": dict(T=3, B=2, I=3, H=4, seed=9, ijfo=True),
    "lstm_stack2_T3_B2_I3_H4": dict(T=3, B=2, I=3, H=4, seed=10, layers=2),
}


def compute(c):
    layers = c.get("layers", 1)
    p = case_inputs(c["T"], c["B"], c["I"], c["H"], c["seed"], layers)
    mask = None
    if c.get("mask"):
        lengths = np.array([c["T"], 1])  # sequence 1 ends after its first step
        t = np.arange(c["T"])[:, None, None]
        mask = (t < lengths[None, :, None]).astype(np.float64) * np.ones((1, 1, c["H"]))
    opt = dict(mask=mask, reverse=c.get("reverse", False), ijfo=c.get("ijfo", False))
    if layers == 1:
        out = oracle.lstm_fwd_bwd(p["x"], p["W"][0], p["b"][0], p["h0"][0], p["c0"][0], p["dy"],
                                  p["dhT"][0], p["dcT"][0], **opt)
        res = {k: out[k] for k in ("y", "hT", "cT", "dx", "dW", "db", "dh0", "dc0")}
    else:
        f = oracle.lstm_stack_fwd(p["x"], p["W"], p["b"], p["h0"], p["c0"], **opt)
        g = oracle.lstm_stack_bwd(p["x"], p["W"], p["h0"], p["c0"], f, p["dy"], p["dhT"], p["dcT"],
                                  **opt)
        res = {"y": f[-1]["y"], "dx": g[0]["dx"]}
        for l in range(layers):
            res[f"hT{l}"] = f[l]["hT"]
            res[f"dW{l}"] = g[l]["dW"]
            res[f"db{l}"] = g[l]["db"]
            res[f"dh0{l}"] = g[l]["dh0"]
    return {k: np.asarray(v).tolist() for k, v in res.items()}


def main():
    for name, c in CASES.items():
        rec = {"case": c, "outputs": compute(c),
               "origin": "fp64 oracle (oracle/lstm_oracle.c), regression record, not a page value"}
        with open(os.path.join(HERE, name + ".json"), "w") as fh:
            json.dump(rec, fh, indent=0)
        print("wrote", name)


if __name__ == "__main__":
    main()
