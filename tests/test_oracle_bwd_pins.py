"""Pins of the oracle's backward pass against facts fixed outside it.

The backward pass is defined by the forward one: its outputs are the partial
derivatives of loss = sum_t <dy_t, y_t> + <dfinal, final_state> with respect
to every forward input.  The pins check it against

- central finite differences of the (separately pinned) forward recurrence,
  element by element on a tiny case and along random directions on a case
  long enough to cross the backward's recomputation segments;
- the derivatives of a one-token sequence, worked out by hand.

Any plausible slip in the adjoint (a dropped term, a wrong sign, an
off-by-one in the decay, a missing chain-rule factor) fails at least one of
them.  No GPU is used.
"""
import numpy as np
import pytest

import oracle

from tests.test_oracle_pins import rand_case, rel

GRADS = {"x": "dx", "dt_raw": "ddt_raw", "dt_bias": "ddt_bias", "A": "dA", "B": "dB", "C": "dC", "D": "dD",
         "init_state": "dinit_state"}


def loss(case, dy, dfinal):
    y, fs = oracle.recurrent(**case)
    return float(np.sum(dy * y) + np.sum(dfinal * fs))


def make(rng, **kw):
    case = rand_case(rng, **kw)
    b, L, H, P = case["x"].shape
    N = case["B"].shape[3]
    dy = rng.standard_normal((b, L, H, P))
    dfinal = rng.standard_normal((b, H, N, P))
    return case, dy, dfinal


# b1: every element of every gradient against a central difference
@pytest.mark.parametrize("G", [1, 2])
def test_backward_elementwise_finite_differences(G):
    rng = np.random.default_rng(40 + G)
    case, dy, dfinal = make(rng, b=2, L=5, H=2, P=3, N=2, G=G)
    grads = oracle.backward(**case, dy=dy, dfinal=dfinal)
    eps = 1e-6
    for name, gname in GRADS.items():
        arr = case[name]
        fd = np.empty_like(arr)
        for i in np.ndindex(arr.shape):
            keep = arr[i]
            arr[i] = keep + eps
            lp = loss(case, dy, dfinal)
            arr[i] = keep - eps
            lm = loss(case, dy, dfinal)
            arr[i] = keep
            fd[i] = (lp - lm) / (2 * eps)
        assert rel(grads[gname], fd) < 1e-6, name


# b2: directional derivatives on a sequence longer than the recomputation segment
@pytest.mark.parametrize("with_init,with_dfinal", [(True, True), (False, False)])
def test_backward_directional_finite_differences(with_init, with_dfinal):
    rng = np.random.default_rng(7)
    case, dy, dfinal = make(rng, b=2, L=150, H=4, P=4, N=3, G=2, with_init=with_init)
    if not with_dfinal:
        dfinal = np.zeros_like(dfinal)
    grads = oracle.backward(**case, dy=dy, dfinal=dfinal if with_dfinal else None)
    eps = 1e-6
    for name, gname in GRADS.items():
        if case[name] is None:
            continue
        for _ in range(2):
            v = rng.standard_normal(case[name].shape)
            base = case[name].copy()
            case[name] = base + eps * v
            lp = loss(case, dy, dfinal)
            case[name] = base - eps * v
            lm = loss(case, dy, dfinal)
            case[name] = base
            fd = (lp - lm) / (2 * eps)
            an = float(np.sum(grads[gname] * v))
            assert abs(an - fd) <= 1e-6 * max(1.0, abs(fd)), (name, an, fd)


# b3: a single token, by hand.  With h = exp(a) h0 + dt B x^T, a = dt A,
# y = C^T h + D x and loss = <dy, y>:
#   dx = dt (B.C) dy + D dy            dB = dt (x.dy) C
#   dC = exp(a) h0 dy + dt (x.dy) B     dD = x.dy
#   dh0 = exp(a) C dy^T
#   d loss/d dt = (B.C)(x.dy) + A exp(a) C^T h0 dy
#   ddt_raw = ddt_bias = that * sigmoid(dt_raw + dt_bias)
#   dA = dt exp(a) C^T h0 dy
def test_backward_single_token_closed_form():
    rng = np.random.default_rng(3)
    P, N = 3, 4
    x, dy = rng.standard_normal(P), rng.standard_normal(P)
    Bv, Cv, h0 = rng.standard_normal(N), rng.standard_normal(N), rng.standard_normal((N, P))
    z, A, D = 0.3, -1.7, 0.6
    dt = np.log1p(np.exp(z))
    e = np.exp(dt * A)
    g = oracle.backward(x=x.reshape(1, 1, 1, P), dt_raw=np.array([[[z]]]), dt_bias=None, A=np.array([A]),
                        B=Bv.reshape(1, 1, 1, N), C=Cv.reshape(1, 1, 1, N), D=np.array([D]),
                        init_state=h0.reshape(1, 1, N, P), dy=dy.reshape(1, 1, 1, P))
    xdy, bc, ch0dy = x @ dy, Bv @ Cv, Cv @ h0 @ dy
    ddt = bc * xdy + A * e * ch0dy
    sig = 1.0 / (1.0 + np.exp(-z))
    np.testing.assert_allclose(g["dx"].ravel(), dt * bc * dy + D * dy, rtol=1e-13)
    np.testing.assert_allclose(g["dB"].ravel(), dt * xdy * Cv, rtol=1e-13)
    np.testing.assert_allclose(g["dC"].ravel(), e * h0 @ dy + dt * xdy * Bv, rtol=1e-13)
    np.testing.assert_allclose(g["dD"], [xdy], rtol=1e-13)
    np.testing.assert_allclose(g["dinit_state"].reshape(N, P), e * np.outer(Cv, dy), rtol=1e-13)
    np.testing.assert_allclose(g["ddt_raw"].ravel(), [ddt * sig], rtol=1e-12)
    np.testing.assert_allclose(g["ddt_bias"], [ddt * sig], rtol=1e-12)
    np.testing.assert_allclose(g["dA"], [dt * e * ch0dy], rtol=1e-12)


# b4: an empty sequence passes dfinal straight through to the initial state
def test_backward_empty_sequence():
    rng = np.random.default_rng(9)
    case, dy, dfinal = make(rng, b=2, L=0, H=2, P=3, N=2, G=1)
    g = oracle.backward(**case, dy=dy, dfinal=dfinal)
    np.testing.assert_array_equal(g["dinit_state"], dfinal)
    assert not np.any(g["dA"]) and not np.any(g["dD"]) and not np.any(g["ddt_bias"])
