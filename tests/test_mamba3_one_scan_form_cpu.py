"""The algebra the one-scan Mamba-3 prefill rests on, checked in float64 on the
CPU against the oracle's sequential recurrence (no GPU).

The head-pair kernel's Mamba-3 form never carries the trapezoid's left end or
turns the state token by token.  It relies on three identities of the
recurrence ("Mamba3", sections "New discretisation scheme" and on
complex-valued SSMs; "Mamba-3 : SSM optimise inference", "Etats complexes via
RoPE"), with Theta_t the running sum of the angles:

  - in the turned frame ~h_t = R(-Theta_t) h_t the recurrence is real, with
    ~B_t = R(-Theta_t) B_t and ~C_t = R(-Theta_t) C_t;
  - token s enters every later state with weight
    w_s = lam_s dt_s + (1 - lam_{s+1}) dt_{s+1}, and its own output with
    lam_s dt_s (the diagonal of the masked matrix);
  - the final state is R(Theta_{L-1}) applied to the turned one, and the
    initial state enters the turned frame unchanged.

Here the masked quadratic form is evaluated with exactly those weights and
compared with the oracle element by element.  A slip in any of them (the
diagonal taking w_s, the left end's weight taken from token s instead of
s + 1, the final state left turned) moves the result by far more than the
bound, which the last test checks."""
import numpy as np
import pytest

import oracle
from mamba_ssd_scan_chunked_b200 import inputs as I


def _turn(v, phi):
    """Pairs (2k, 2k+1) of the last axis turned counter-clockwise by phi[..., k]."""
    out = v.copy()
    c, s = np.cos(phi), np.sin(phi)
    u, w = v[..., 0::2], v[..., 1::2]
    out[..., 0::2] = c * u - s * w
    out[..., 1::2] = s * u + c * w
    return out


def one_scan_form(x, dt_raw, dt_bias, A, B, C, D, lam, theta, h0, diag="lam_dt", left="next", turn_back=True):
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    hpg = H // G
    Th = np.cumsum(theta, axis=1)                       # [b, L, G, N/2]
    Bt, Ct = _turn(B, -Th), _turn(C, -Th)
    dt = np.log1p(np.exp(dt_raw + dt_bias))             # [b, L, H]
    a = dt * A
    lam_n = np.concatenate([lam[:, 1:], np.ones_like(lam[:, :1])], axis=1)
    dt_n = np.concatenate([dt[:, 1:], np.zeros_like(dt[:, :1])], axis=1)
    w = lam * dt + ((1 - lam_n) * dt_n if left == "next" else (1 - lam) * dt)
    own = lam * dt if diag == "lam_dt" else w
    y = np.empty_like(x)
    fs = np.empty((b, H, N, P))
    for bi in range(b):
        for h in range(H):
            g = h // hpg
            cum = np.cumsum(a[bi, :, h])
            S = Ct[bi, :, g] @ Bt[bi, :, g].T               # [L, L]: ~C_t . ~B_s
            dec = np.exp(cum[:, None] - cum[None, :])       # exp(sum_{s<u<=t} a_u)
            M = np.tril(S * dec * w[bi, :, h][None, :], -1)
            M[np.diag_indices(L)] = np.diag(S) * own[bi, :, h]
            y[bi, :, h] = M @ x[bi, :, h] + (Ct[bi, :, g] * np.exp(cum)[:, None]) @ h0[bi, h] + D[h] * x[bi, :, h]
            wdec = np.exp(cum[-1] - cum) * w[bi, :, h]      # weight of token s in the last state
            S_turned = Bt[bi, :, g].T @ (wdec[:, None] * x[bi, :, h]) + np.exp(cum[-1]) * h0[bi, h]
            fs[bi, h] = (_turn(S_turned.T, Th[bi, -1, g]).T if turn_back else S_turned)
    return y, fs


def _case(b=2, L=37, H=4, P=3, N=6, G=2, seed=5):
    inp = I.prefill_inputs(b, L, H, P, N, G, seed, I.F32)
    ex = I.draw_mamba3_extras(b, L, H, G, N, seed)
    f = {k: I.to_f64(v) for k, v in inp.items()}
    lam, theta = I.to_f64(ex["lam"]), I.to_f64(ex["theta"])
    h0 = 0.3 * np.random.default_rng([seed, 1]).standard_normal((b, H, N, P))
    y_ref, fs_ref = oracle.mamba3_recurrent(f["x"], f["dt_raw"], f["dt_bias"], f["A"], f["B"], f["C"], f["D"],
                                            lam=lam, theta=theta, init_state=h0)
    args = (f["x"], f["dt_raw"], f["dt_bias"], f["A"], f["B"], f["C"], f["D"], lam, theta, h0)
    return args, y_ref, fs_ref


def _m(g, r):
    return float(np.max(np.abs(g - r)) / np.sqrt(np.mean(r * r)))


def test_one_scan_form_equals_the_recurrence():
    args, y_ref, fs_ref = _case()
    y, fs = one_scan_form(*args)
    assert _m(y, y_ref) < 1e-12
    assert _m(fs, fs_ref) < 1e-12


@pytest.mark.parametrize("slip", [dict(diag="w"), dict(left="same"), dict(turn_back=False)])
def test_each_slip_in_the_form_is_seen(slip):
    args, y_ref, fs_ref = _case()
    y, fs = one_scan_form(*args, **slip)
    assert max(_m(y, y_ref), _m(fs, fs_ref)) > 1e-3
