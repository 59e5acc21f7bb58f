"""GPU parity of ssd_replay_step (decode from a checkpoint plus a buffer of the
tokens after it) against the float64 oracle's sequential recurrence.

The oracle steps the plain recurrence token by token; where the library stores
the checkpoint in bf16 -- at the steps that fold the buffer into it -- the
oracle rounds its state to bf16 at the same steps.  Every step's y is
compared, and at every fold the checkpoint itself."""
import numpy as np
import pytest

import oracle
from mamba_ssd_scan_chunked_b200 import inputs as I
from mamba_ssd_scan_chunked_b200 import ssd
from tests.gpu_util import TOL_BF16, TOL_F32, bf16_state_metric, metric, to_dev, to_host64, torch

pytestmark = pytest.mark.gpu


def run_case(b, H, P, N, G, K, io, state, nsteps, seed=21):
    t = torch()
    params = I.draw_head_params(H, seed=seed)
    st0 = np.stack([I.draw_decode_state(i, H, P, N, seed=seed + 1, dtype=state) for i in range(b)])
    steps = [I.draw_decode_step(s, b, H, P, N, G, seed=seed + 2, dtype=io) for s in range(nsteps)]
    ckpt = to_dev(st0)
    prm = {k: to_dev(v) for k, v in params.items()}
    dev_steps = [{k: to_dev(v) for k, v in s.items()} for s in steps]
    buf = ssd.replay_buffer(ckpt, dev_steps[0]["x"], dev_steps[0]["B"], K)
    ref = I.to_f64(st0).copy()
    f = {k: I.to_f64(v) for k, v in params.items()}
    fill = 0
    worst_y, worst_state, folds = 0.0, 0.0, 0
    for s, (hs, ds) in enumerate(zip(steps, dev_steps)):
        folding = fill == K - 1
        y, fill = ssd.replay_step(ckpt, buf, fill, K, ds["x"], ds["dt_raw"], prm["dt_bias"], prm["A"], ds["B"],
                                  ds["C"], prm["D"], y_dtype=t.float32)
        g = {k: I.to_f64(v) for k, v in hs.items()}
        y_ref = oracle.decode_step(ref, g["x"], g["dt_raw"], f["dt_bias"], f["A"], g["B"], g["C"], f["D"])
        if folding and state == I.BF16:
            ref[...] = oracle.round_bf16(ref)
        worst_y = max(worst_y, metric(to_host64(y), y_ref))
        if folding:
            got = to_host64(ckpt)
            worst_state = max(worst_state, (bf16_state_metric if state == I.BF16 else metric)(got, ref))
            folds += 1
    t.cuda.synchronize()
    assert ssd.ssd_get_device_error(0)[0] == 0
    return worst_y, worst_state, folds


@pytest.mark.parametrize("b,H,P,N,G,K,io,state", [
    (3, 4, 64, 128, 2, 16, I.BF16, I.F32),     # the decode workload's head shape, full buffer
    (2, 6, 32, 16, 3, 4, I.F32, I.F32),        # fp32 throughout
    (2, 4, 128, 64, 1, 8, I.BF16, I.BF16),     # bf16 checkpoint, rounded at folds only
    (1, 2, 8, 8, 2, 1, I.F32, I.F32),          # capacity 1: every step folds (the plain step)
    (2, 4, 16, 256, 4, 5, I.BF16, I.F32),      # dstate 256, odd capacity
    (1, 3, 64, 256, 1, 16, I.BF16, I.BF16),    # dstate 256, full buffer (68 KB of flush smem)
])
def test_replay_matches_sequential_recurrence(b, H, P, N, G, K, io, state):
    nsteps = 2 * K + 3                         # two folds and a partly filled buffer
    worst_y, worst_state, folds = run_case(b, H, P, N, G, K, io, state, nsteps)
    assert folds == 2 if K > 1 else folds == nsteps
    tol = TOL_F32 if (io == I.F32 and state == I.F32) else TOL_BF16
    assert worst_y <= tol
    assert worst_state <= tol


def test_capacity_one_equals_state_update():
    """Capacity 1 folds every step: the same recurrence as ssd_state_update."""
    t = torch()
    b, H, P, N, G = 2, 4, 64, 32, 2
    params = I.draw_head_params(H, seed=5)
    st0 = np.stack([I.draw_decode_state(i, H, P, N, seed=6, dtype=I.F32) for i in range(b)])
    prm = {k: to_dev(v) for k, v in params.items()}
    s_plain, s_replay = to_dev(st0), to_dev(st0)
    buf = None
    for s in range(5):
        d = {k: to_dev(v) for k, v in I.draw_decode_step(s, b, H, P, N, G, seed=7, dtype=I.F32).items()}
        if buf is None:
            buf = ssd.replay_buffer(s_replay, d["x"], d["B"], 1)
        y1 = ssd.state_update(s_plain, d["x"], d["dt_raw"], prm["dt_bias"], prm["A"], d["B"], d["C"], prm["D"])
        y2, fill = ssd.replay_step(s_replay, buf, 0, 1, d["x"], d["dt_raw"], prm["dt_bias"], prm["A"], d["B"],
                                   d["C"], prm["D"])
        assert fill == 0
        assert metric(to_host64(y2), to_host64(y1)) <= 1e-5
    # fp32 either way; only the rounding order differs (alpha h + (beta B_n) x_p
    # here, one fma of exp(dt A) h and dt B_n x_p there), over five steps
    assert metric(to_host64(s_replay), to_host64(s_plain)) <= 1e-5


def test_rollback_by_lowering_fill():
    """Speculative decoding: the checkpoint is only read until the buffer fills,
    so dropping the last k buffered tokens is a call with fill - k.  Steps 0..5
    are taken, steps 4 and 5 are rejected, and two other tokens follow; the
    outputs must be the oracle's for the accepted sequence 0..3, 6, 7."""
    t = torch()
    b, H, P, N, G, K = 2, 4, 64, 128, 2, 16
    params = I.draw_head_params(H, seed=71)
    st0 = np.stack([I.draw_decode_state(i, H, P, N, seed=72, dtype=I.F32) for i in range(b)])
    steps = [I.draw_decode_step(s, b, H, P, N, G, seed=73, dtype=I.BF16) for s in range(8)]
    ckpt = to_dev(st0)
    prm = {k: to_dev(v) for k, v in params.items()}
    dev = [{k: to_dev(v) for k, v in s.items()} for s in steps]
    buf = ssd.replay_buffer(ckpt, dev[0]["x"], dev[0]["B"], K)

    def step(i, fill):
        d = dev[i]
        return ssd.replay_step(ckpt, buf, fill, K, d["x"], d["dt_raw"], prm["dt_bias"], prm["A"], d["B"], d["C"],
                               prm["D"], y_dtype=t.float32)

    fill = 0
    for i in range(6):                          # 0..3 accepted, 4 and 5 speculative
        _, fill = step(i, fill)
    fill -= 2                                   # reject 4 and 5
    ys = [step(i, f)[0] for i, f in ((6, fill), (7, fill + 1))]
    ref = I.to_f64(st0).copy()
    f = {k: I.to_f64(v) for k, v in params.items()}
    y_ref = None
    for i in (0, 1, 2, 3, 6, 7):
        g = {k: I.to_f64(v) for k, v in steps[i].items()}
        y_ref = oracle.decode_step(ref, g["x"], g["dt_raw"], f["dt_bias"], f["A"], g["B"], g["C"], f["D"])
        if i == 6:
            y6_ref = y_ref
    assert metric(to_host64(ys[0]), y6_ref) <= TOL_BF16
    assert metric(to_host64(ys[1]), y_ref) <= TOL_BF16
