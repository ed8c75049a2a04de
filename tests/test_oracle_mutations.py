"""The oracle's pins are sensitive: each planted mistake below (a dropped term, a
wrong sign or index, a doubled forget factor, a transposed operand) is compiled
into a throw-away copy of the oracle on the CPU, and the finite-difference pin
must reject it.  The mistakes are planted in the oracle only, never in a kernel.
"""
import os

import numpy as np
import pytest

import oracle
from tests.test_oracle import fd_max_error, random_case, random_mask

SRC = os.path.join(os.path.dirname(oracle.__file__), "lstm_oracle.c")

MUTATIONS = {
    # forget factor applied twice to the carried cell gradient (backward step 2)
    "double_forget": ("double dc = dh * o_ * (1.0 - tc * tc) + m * dc_next[j];",
                      "double dc = dh * o_ * (1.0 - tc * tc) + m * dc_next[j] * f_;"),
    # dL_t/dh_t dropped from step 1
    "drop_dy": ("double dh_tot = (dyt ? dyt[j] : 0.0) + dh_next[j];",
                "double dh_tot = dh_next[j];"),
    # sign error in the forget-gate derivative (step 3)
    "sign_df": ("double d_f = dc * c_prev * f_ * (1.0 - f_);",
                "double d_f = dc * c_prev * f_ * (1.0 + f_);"),
    # i and f gradients stored in each other's rows
    "swap_rows": ("dGt[j] = d_i;\n                dGt[BF + j] = d_f;",
                  "dGt[j] = d_f;\n                dGt[BF + j] = d_i;"),
    # c_t used where c_{t-1} belongs in the forget-gate gradient
    "wrong_cprev": ("double d_f = dc * c_prev * f_ * (1.0 - f_);",
                    "double d_f = dc * c_ * f_ * (1.0 - f_);"),
    # delta c_prev loses its forget factor (step 5)
    "no_forget_carry": ("dc_next[j] = dc * f_ + (1.0 - m) * dc_next[j];",
                        "dc_next[j] = dc + (1.0 - m) * dc_next[j];"),
    # h-part and x-part of dz exchanged (transposed operand of W^T dG)
    "dz_parts_swapped": ("dxt[k] = dz[H + k];", "dxt[k] = dz[k % (H > 0 ? H : 1)];"),
    # dW accumulates x_{t-1} instead of x_t
    "dW_wrong_x": ("const double *xt = x + ((long)t * B + n) * I;\n                    if (hp)",
                   "const double *xt = x + ((long)(t > 0 ? t - 1 : 0) * B + n) * I;\n                    if (hp)"),
    # tanh(c) replaced by c in the output-gate gradient
    "do_missing_tanh": ("double d_o = dh * tc * o_ * (1.0 - o_);",
                        "double d_o = dh * c_ * o_ * (1.0 - o_);"),
    # padding does not pass delta h on to h_{t-1} (variable-length mask)
    "mask_no_h_pass": ("dh_pass[j] = (1.0 - m) * dh_tot;", "dh_pass[j] = 0.0;"),
    # padding updates the cell state anyway (variable-length mask, forward)
    "mask_c_moves": ("c_ = mt[j] * c_ + (1.0 - mt[j]) * cprev[j];", "c_ = c_;"),
    # reverse direction: the previous cell state of the forget-gate gradient
    # taken at the step's own time instead of time t + 1 (stays in bounds, unlike
    # the forward direction's neighbour t - 1, which runs off the array at t = 0)
    "reverse_cprev": ("const int tp = reverse ? t + 1 : t - 1;        /* time of step s - 1 */",
                      "const int tp = reverse ? t : t - 1;"),
}

# mutations that only a masked case can reveal
MASKED = {"mask_no_h_pass", "mask_c_moves"}
# and only a reverse-direction case
REVERSE = {"reverse_cprev"}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    lib = oracle.load_variant(oracle.compile_source(str(path), str(tmp_path / "mutant.so")))
    p, g = random_case(3, 2, 3, 4, seed=99)
    mask = random_mask(3, 2, 4, seed=5) if name in MASKED else None
    rev = name in REVERSE
    assert fd_max_error(p, g, lib=lib, mask=mask, reverse=rev) > 1e-3, \
        f"mutation {name} slipped through"
    # the unmutated oracle passes the same pin
    assert fd_max_error(p, g, mask=mask, reverse=rev) < 1e-6
