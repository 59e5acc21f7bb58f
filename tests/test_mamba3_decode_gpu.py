"""GPU parity of ssd_state_update_mamba3 (the Mamba-3 decode step: trapezoidal
input mixed by lam, state pairs turned by theta) against the float64 oracle's
Mamba-3 step, over 32 consecutive tokens from a random state: every step's y and
the final state, fp32 and bf16 states, with and without the mix and the angles.
"Mamba3" (Telegram post), section "New discretisation scheme" and the section
on the complex-valued SSM; "Mamba-3 : SSM optimise inference", section "Etats
complexes via RoPE"."""
import numpy as np
import pytest

import oracle
from mamba_ssd_scan_chunked_b200 import inputs as I
from mamba_ssd_scan_chunked_b200 import ssd
from tests.gpu_util import TOL_BF16, TOL_F32, bf16_state_metric, metric, to_dev, to_host64, torch

pytestmark = pytest.mark.gpu

T = 32


def run(b, H, P, N, G, io, state_dtype, with_lam, with_theta, seed=80):
    t = torch()
    params = I.draw_head_params(H, seed=seed)
    st0 = np.stack([I.draw_decode_state(i, H, P, N, seed=seed + 1, dtype=state_dtype) for i in range(b)])
    steps = [I.draw_decode_step(k, b, H, P, N, G, seed=seed + 2, dtype=io) for k in range(T)]
    ex = I.draw_mamba3_extras(b, T, H, G, N, seed + 3)      # lam [b,T,H], theta [b,T,G,N/2]
    lam = [np.ascontiguousarray(ex["lam"][:, k]) if with_lam else None for k in range(T)]
    theta = [np.ascontiguousarray(ex["theta"][:, k]) if with_theta else None for k in range(T)]

    # GPU: the caller keeps the previous token's x and B
    state = to_dev(st0)
    prm = {k: to_dev(v) for k, v in params.items()}
    ys, prev = [], None
    for k, s in enumerate(steps):
        d = {kk: to_dev(v) for kk, v in s.items()}
        y = ssd.state_update_mamba3(state, d["x"], d["dt_raw"], prm["dt_bias"], prm["A"], d["B"], d["C"], prm["D"],
                                    x_prev=prev["x"] if prev else None, B_prev=prev["B"] if prev else None,
                                    lam=to_dev(lam[k]) if with_lam else None,
                                    theta=to_dev(theta[k]) if with_theta else None, y_dtype=t.float32)
        ys.append(to_host64(y))
        prev = d
    t.cuda.synchronize()
    s_gpu = to_host64(state)

    # oracle: its in-place previous-token buffers start at zero
    st = I.to_f64(st0).copy()
    Bp = np.zeros((b, G, N))
    xp = np.zeros((b, H, P))
    f = {k: I.to_f64(v) for k, v in params.items()}
    ys_ref = []
    for k, s in enumerate(steps):
        g = {kk: I.to_f64(v) for kk, v in s.items()}
        ys_ref.append(oracle.mamba3_decode_step(st, Bp, xp, g["x"], g["dt_raw"], f["dt_bias"], f["A"], g["B"],
                                                g["C"], f["D"], lam=lam[k], theta=theta[k]))
        if state_dtype == I.BF16:      # the state is stored in bf16 after every step
            st[...] = oracle.round_bf16(st)
    return ys, s_gpu, ys_ref, st


@pytest.mark.parametrize("b,H,P,N,G", [(3, 4, 64, 128, 2), (2, 6, 32, 16, 3), (4, 8, 64, 64, 1), (2, 4, 128, 32, 4)])
@pytest.mark.parametrize("io,state_dtype", [(I.F32, I.F32), (I.BF16, I.F32), (I.BF16, I.BF16)])
def test_mamba3_decode_matches_oracle(b, H, P, N, G, io, state_dtype):
    ys, s_gpu, ys_ref, s_ref = run(b, H, P, N, G, io, state_dtype, True, True)
    tol = TOL_F32 if io == I.F32 and state_dtype == I.F32 else TOL_BF16
    for y, yr in zip(ys, ys_ref):
        assert metric(y, yr) <= tol
    state_metric = bf16_state_metric if state_dtype == I.BF16 else metric
    assert state_metric(s_gpu, s_ref) <= tol


@pytest.mark.parametrize("with_lam,with_theta", [(True, False), (False, True)])
def test_mamba3_decode_mix_or_rotation_alone(with_lam, with_theta):
    ys, s_gpu, ys_ref, s_ref = run(2, 8, 64, 128, 2, I.F32, I.F32, with_lam, with_theta, seed=90)
    for y, yr in zip(ys, ys_ref):
        assert metric(y, yr) <= TOL_F32
    assert metric(s_gpu, s_ref) <= TOL_F32


def test_mamba3_decode_without_extensions_is_the_plain_step():
    """lam = 1 and theta = 0: the state update of ssd_state_update, bit for bit."""
    t = torch()
    b, H, P, N, G = 4, 8, 64, 128, 2
    params = {k: to_dev(v) for k, v in I.draw_head_params(H, seed=95).items()}
    st0 = to_dev(np.stack([I.draw_decode_state(i, H, P, N, seed=96, dtype=I.F32) for i in range(b)]))
    s1, s2 = st0.clone(), st0.clone()
    for k in range(4):
        d = {kk: to_dev(v) for kk, v in I.draw_decode_step(k, b, H, P, N, G, seed=97, dtype=I.BF16).items()}
        args = (d["x"], d["dt_raw"], params["dt_bias"], params["A"], d["B"], d["C"], params["D"])
        y1 = ssd.state_update(s1, *args, y_dtype=t.float32)
        y2 = ssd.state_update_mamba3(s2, *args, y_dtype=t.float32)
        t.cuda.synchronize()
        assert t.equal(s1, s2)
        assert metric(to_host64(y2), to_host64(y1)) <= 1e-5   # the same terms summed in another fp32 order
