"""Write tests/golden/oracle_tiny.json: a regression fixture of the float64 oracle.

Calls only ``oracle/`` (and the seeded input generator).  The pages print no
worked example, so this fixture does not pin the oracle to the pages -- the
pins in tests/test_oracle_pins.py do that.  It freezes the oracle's outputs on
one tiny seeded case so that any later change to the oracle's arithmetic shows
up as a failing test (and must then name the passage that justifies it).

Case: batch 2, seqlen 24, 4 heads, P=8, N=4, 2 groups, bf16-rounded inputs,
seed 7, random N(0, 0.5^2) initial state from default_rng([7, 9]).
Recurrence per head: dt = softplus(dt_raw + dt_bias), h_t = exp(dt A) h_{t-1}
+ dt B_t x_t^T, y_t = C_t^T h_t + D x_t ("Mamba3", Telegram post, sections on
Mamba-2's scalar transition and on the ZOH/Euler discretisation).
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from mamba_ssd_scan_chunked_b200 import inputs as I  # noqa: E402

SHAPE = dict(batch=2, seqlen=24, nheads=4, headdim=8, dstate=4, ngroups=2, seed=7)


def case():
    s = SHAPE
    inp = I.prefill_inputs(s["batch"], s["seqlen"], s["nheads"], s["headdim"], s["dstate"], s["ngroups"],
                           s["seed"], I.BF16)
    h0 = np.random.default_rng([7, 9]).normal(0, 0.5, (s["batch"], s["nheads"], s["dstate"], s["headdim"]))
    return {k: I.to_f64(v) for k, v in inp.items()}, h0


def main():
    inp, h0 = case()
    y, fs = oracle.recurrent(inp["x"], inp["dt_raw"], inp["dt_bias"], inp["A"], inp["B"], inp["C"], inp["D"],
                             init_state=h0)
    out = {"shape": SHAPE, "source": "oracle.recurrent (float64)",
           "y": y.ravel().tolist(), "final_state": fs.ravel().tolist()}
    with open(os.path.join(HERE, "oracle_tiny.json"), "w") as f:
        json.dump(out, f)


if __name__ == "__main__":
    main()
