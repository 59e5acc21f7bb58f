"""Pins of the oracle's Mamba-3 recurrence (exponential-trapezoidal input and
rotational state) against facts fixed outside it: the Mamba-2 recurrence it
reduces to, closed forms of impulse and step responses, and invariances of
rotations.  No GPU is used."""
import numpy as np
import pytest

import oracle

from tests.test_oracle_pins import rand_case, rel


def softplus(z):
    return np.log1p(np.exp(z))


def mamba3_case(rng, b=2, L=29, H=4, P=3, N=6, G=2, with_init=True):
    c = rand_case(rng, b=b, L=L, H=H, P=P, N=N, G=G, with_init=with_init)
    c["lam"] = rng.uniform(0.0, 1.0, (b, L, H))
    c["theta"] = rng.uniform(-np.pi, np.pi, (b, L, G, N // 2))
    return c


# m1: lam = 1 and theta = 0 are Mamba-2's recurrence (Euler input, real state)
@pytest.mark.parametrize("explicit", [False, True])
def test_mamba3_reduces_to_mamba2(explicit):
    rng = np.random.default_rng(1)
    c = mamba3_case(rng)
    lam, theta = c.pop("lam"), c.pop("theta")
    if explicit:
        lam, theta = np.ones_like(lam), np.zeros_like(theta)
    else:
        lam, theta = None, None
    y3, f3 = oracle.mamba3_recurrent(**c, lam=lam, theta=theta)
    y2, f2 = oracle.recurrent(**c)
    assert rel(y3, y2) < 1e-13 and rel(f3, f2) < 1e-13


def scalar_case(L, dt_raw, A, lam, x, Bv, theta=None, N=1, Cv=None):
    """One head, one group, headdim 1, constant dt_raw."""
    Cv = np.ones((L, N)) if Cv is None else Cv
    return oracle.mamba3_recurrent(
        x=np.asarray(x, float).reshape(1, L, 1, 1), dt_raw=np.full((1, L, 1), dt_raw), dt_bias=None,
        A=np.array([A]), B=np.asarray(Bv, float).reshape(1, L, 1, N), C=Cv.reshape(1, L, 1, N), D=None,
        lam=np.full((1, L, 1), lam), theta=None if theta is None else np.asarray(theta, float).reshape(1, L, 1, N // 2))


# m2: impulse through the trapezoid: h_0 = lam dt B_0 and, for t >= 1, the
# left end adds (1 - lam) dt B_0 before the transition, so h_t = a^t dt B_0
def test_trapezoid_impulse_response():
    L, z, A, lam, b0 = 12, 0.4, -0.9, 0.3, 1.7
    dt = softplus(z)
    a = np.exp(dt * A)
    x = np.zeros(L)
    x[0] = 1.0
    y, _ = scalar_case(L, z, A, lam, x, np.full(L, b0))
    want = np.array([lam * dt * b0] + [a ** t * dt * b0 for t in range(1, L)])
    np.testing.assert_allclose(y.ravel(), want, rtol=1e-13)


# m3: step input x = 1, B = 1: h_0 = lam dt, h_t = a h_{t-1} + dt (a (1 - lam) + lam)
def test_trapezoid_step_response_closed_form():
    L, z, A, lam = 40, -0.2, -1.3, 0.65
    dt = softplus(z)
    a = np.exp(dt * A)
    c = dt * (a * (1 - lam) + lam)
    h_inf = c / (1 - a)
    y, _ = scalar_case(L, z, A, lam, np.ones(L), np.ones(L))
    t = np.arange(L)
    want = h_inf + (lam * dt - h_inf) * a ** t
    np.testing.assert_allclose(y.ravel(), want, rtol=1e-12)


# m4: a rotating pair: impulse B_0 = (1, 0) under a constant angle per step gives
# h_t = a^t dt (cos t th, sin t th) for t >= 1 (any lam), read out by C = (c0, c1)
@pytest.mark.parametrize("lam", [1.0, 0.4])
def test_rotation_impulse_response(lam):
    L, z, A, th = 15, 0.1, -0.5, 0.7
    dt = softplus(z)
    a = np.exp(dt * A)
    x = np.zeros(L)
    x[0] = 1.0
    Bv = np.zeros((L, 2))
    Bv[0] = (1.0, 0.0)
    c0, c1 = 0.8, -1.1
    Cv = np.tile([c0, c1], (L, 1))
    y, fs = scalar_case(L, z, A, lam, x, Bv, theta=np.full(L, th), N=2, Cv=Cv)
    t = np.arange(1, L)
    want = np.concatenate([[lam * dt * c0], a ** t * dt * (c0 * np.cos(t * th) + c1 * np.sin(t * th))])
    np.testing.assert_allclose(y.ravel(), want, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(fs.ravel(), a ** (L - 1) * dt * np.array([np.cos((L - 1) * th), np.sin((L - 1) * th)]),
                               rtol=1e-12)


def rotate_pairs(v, phi):
    """Rotate the pairs (2k, 2k+1) of the last axis by phi[k]."""
    out = v.copy()
    c, s = np.cos(phi), np.sin(phi)
    u, w = v[..., 0::2], v[..., 1::2]
    out[..., 0::2] = c * u - s * w
    out[..., 1::2] = s * u + c * w
    return out


# m5: planar rotations commute, so rotating every B and C by the same angles
# leaves y unchanged (zero initial state) and rotates the final state's rows
def test_common_rotation_of_B_and_C_is_invisible():
    rng = np.random.default_rng(2)
    c = mamba3_case(rng, with_init=False)
    phi = rng.uniform(-np.pi, np.pi, c["B"].shape[3] // 2)
    y1, f1 = oracle.mamba3_recurrent(**c)
    c2 = dict(c, B=rotate_pairs(c["B"], phi), C=rotate_pairs(c["C"], phi))
    y2, f2 = oracle.mamba3_recurrent(**c2)
    assert rel(y2, y1) < 1e-12
    f1r = np.swapaxes(rotate_pairs(np.swapaxes(f1, 2, 3), phi), 2, 3)
    assert rel(f2, f1r) < 1e-12


# m6: the first step's rotation acts on the (zero) state before any input, so
# the angle of token 0 cannot matter without an initial state; with one it does
def test_first_angle_acts_on_the_state_only():
    rng = np.random.default_rng(3)
    c = mamba3_case(rng, with_init=False)
    y1, _ = oracle.mamba3_recurrent(**c)
    th = c["theta"].copy()
    th[:, 0] += 1.0
    y2, _ = oracle.mamba3_recurrent(**dict(c, theta=th))
    assert rel(y2, y1) < 1e-13
    c = mamba3_case(rng, with_init=True)
    y3, _ = oracle.mamba3_recurrent(**c)
    y4, _ = oracle.mamba3_recurrent(**dict(c, theta=th))
    assert rel(y4, y3) > 1e-3


# m7: every head of a group turns with the group's angles: zero angles on group 1
# give Mamba-2 with the trapezoid for its heads whatever group 0 does
def test_angles_follow_the_group_map():
    rng = np.random.default_rng(4)
    c = mamba3_case(rng, H=4, G=2)
    th = c["theta"].copy()
    th[:, :, 1] = 0.0
    y_rot, _ = oracle.mamba3_recurrent(**dict(c, theta=th))
    y_flat, _ = oracle.mamba3_recurrent(**dict(c, theta=None))
    assert rel(y_rot[:, :, 2:], y_flat[:, :, 2:]) < 1e-13      # heads 2, 3 read group 1
    assert rel(y_rot[:, :, :2], y_flat[:, :, :2]) > 1e-3


# m8: the decode step (state + the previous token's B and x) stepped over a
# sequence reproduces the sequence recurrence token by token
def test_mamba3_decode_steps_equal_the_recurrence():
    rng = np.random.default_rng(6)
    c = mamba3_case(rng, b=2, L=17, H=4, P=3, N=6, G=2)
    y_ref, f_ref = oracle.mamba3_recurrent(**c)
    b, L, H, P = c["x"].shape
    G, N = c["B"].shape[2:]
    st = c["init_state"].copy()
    Bp, xp = np.zeros((b, G, N)), np.zeros((b, H, P))
    for t in range(L):
        y = oracle.mamba3_decode_step(st, Bp, xp, c["x"][:, t], c["dt_raw"][:, t], c["dt_bias"], c["A"],
                                      c["B"][:, t], c["C"][:, t], c["D"], c["lam"][:, t], c["theta"][:, t])
        assert rel(y, y_ref[:, t]) < 1e-12
    assert rel(st, f_ref) < 1e-12
