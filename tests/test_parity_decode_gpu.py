"""GPU parity of ssd_state_update (decode) against the float64 oracle, and the
prefill/decode cross-path invariants."""
import numpy as np
import pytest

import oracle
from mamba_ssd_scan_chunked_b200 import inputs as I
from mamba_ssd_scan_chunked_b200 import ssd
from tests.gpu_util import (TOL_BF16, TOL_F32, bf16_state_metric, gpu_prefill, metric, oracle_prefill,
                            random_state, to_dev, to_host64, torch)

pytestmark = pytest.mark.gpu


def run_decode(state0, steps, params, y_dtype="f32"):
    """GPU: `steps` consecutive ssd_state_update calls from state0 (storage array).
    Returns (list of y per step as float64, final state as float64)."""
    t = torch()
    st = to_dev(state0)
    prm = {k: to_dev(v) for k, v in params.items()}
    ys = []
    for s in steps:
        d = {k: to_dev(v) for k, v in s.items()}
        y = ssd.state_update(st, d["x"], d["dt_raw"], prm["dt_bias"], prm["A"], d["B"], d["C"], prm["D"],
                             y_dtype=t.float32 if y_dtype == "f32" else t.bfloat16)
        ys.append(to_host64(y))
    t.cuda.synchronize()
    return ys, to_host64(st)


def oracle_decode(state0, steps, params, round_bf16):
    st = I.to_f64(state0).copy()
    ys = []
    f = {k: I.to_f64(v) for k, v in params.items()}
    for s in steps:
        g = {k: I.to_f64(v) for k, v in s.items()}
        ys.append(oracle.decode_step(st, g["x"], g["dt_raw"], f["dt_bias"], f["A"], g["B"], g["C"], f["D"],
                                     round_state_bf16=round_bf16))
    return ys, st


@pytest.mark.parametrize("b,H,P,N,G", [(3, 4, 64, 128, 2), (2, 6, 32, 16, 3), (4, 8, 64, 64, 1),
                                       (1, 2, 128, 256, 2), (2, 4, 8, 8, 4), (2, 3, 24, 32, 1),
                                       (1, 3, 256, 64, 1), (3, 5, 16, 24, 5)])
@pytest.mark.parametrize("io,state", [(I.F32, I.F32), (I.BF16, I.F32), (I.BF16, I.BF16)])
def test_decode_matches_oracle(b, H, P, N, G, io, state):
    params = I.draw_head_params(H, seed=7)
    st0 = np.stack([I.draw_decode_state(i, H, P, N, seed=8, dtype=state) for i in range(b)])
    steps = [I.draw_decode_step(t, b, H, P, N, G, seed=9, dtype=io) for t in range(6)]
    ys, s_gpu = run_decode(st0, steps, params)
    ys_ref, s_ref = oracle_decode(st0, steps, params, round_bf16=(state == I.BF16))
    tol = TOL_F32 if (io == I.F32 and state == I.F32) else TOL_BF16
    for y, yr in zip(ys, ys_ref):
        assert metric(y, yr) <= tol
    state_metric = bf16_state_metric if state == I.BF16 else metric
    assert state_metric(s_gpu, s_ref) <= tol


def test_prefill_one_token_equals_decode_step():
    """prefill(L=1, init=s) == state_update(s) (both paths, same inputs)."""
    b, H, P, N, G = 2, 4, 64, 128, 2
    inp = I.prefill_inputs(b, 1, H, P, N, G, 13, I.BF16)
    h0 = random_state((b, H, N, P), 14, I.F32, std=0.1)
    y_p, f_p = gpu_prefill(inp, 256, h0)
    step = {"x": inp["x"][:, 0], "dt_raw": inp["dt_raw"][:, 0], "B": inp["B"][:, 0], "C": inp["C"][:, 0]}
    params = {k: inp[k] for k in ("dt_bias", "A", "D")}
    ys, s_d = run_decode(h0, [step], params)
    assert metric(y_p[:, 0], ys[0]) <= 1e-3
    assert metric(f_p, s_d) <= 1e-3


def test_prefill_equals_decode_steps():
    """prefill(L) == L decode steps from the same initial state."""
    b, L, H, P, N, G = 2, 300, 4, 64, 128, 2
    inp = I.prefill_inputs(b, L, H, P, N, G, 15, I.BF16)
    h0 = random_state((b, H, N, P), 16, I.F32, std=0.1)
    y_p, f_p = gpu_prefill(inp, 256, h0)
    steps = [{"x": np.ascontiguousarray(inp["x"][:, t]), "dt_raw": np.ascontiguousarray(inp["dt_raw"][:, t]),
              "B": np.ascontiguousarray(inp["B"][:, t]), "C": np.ascontiguousarray(inp["C"][:, t])}
             for t in range(L)]
    params = {k: inp[k] for k in ("dt_bias", "A", "D")}
    ys, s_d = run_decode(h0, steps, params)
    y_ref, f_ref = oracle_prefill(inp, h0)
    assert metric(np.stack(ys, axis=1), y_ref) <= TOL_BF16
    assert metric(y_p, np.stack(ys, axis=1)) <= TOL_BF16
    assert metric(f_p, s_d) <= TOL_BF16
