"""Pins of the float64 oracle against facts fixed outside the oracle itself.

Each test checks the oracle against a closed form, a textbook special case, an
invariant of the mathematics, or another contraction order of the same
semiseparable matrix ("Mamba-2 vs Transformers / SSD", section "Mamba-2 and the
SSD paper: what changed in practice").  Together they make a plausible slip in
the oracle (a dropped term, a wrong sign or index, a transposed operand, an
off-by-one in the decay cumsum, the state read before instead of after the
update) fail at least one test.  No GPU is used.
"""
import math

import numpy as np
import pytest

import oracle
from mamba_ssd_scan_chunked_b200 import inputs as I


def rand_case(rng, b=2, L=37, H=4, P=5, N=6, G=2, with_init=True, a_scale=1.0):
    x = rng.standard_normal((b, L, H, P))
    dt_raw = rng.standard_normal((b, L, H))
    dt_bias = np.log(np.expm1(rng.uniform(1e-2, 0.5, H)))
    A = -rng.uniform(0.5, 4.0, H) * a_scale
    B = rng.standard_normal((b, L, G, N))
    C = rng.standard_normal((b, L, G, N))
    D = rng.standard_normal(H)
    h0 = rng.standard_normal((b, H, N, P)) if with_init else None
    return dict(x=x, dt_raw=dt_raw, dt_bias=dt_bias, A=A, B=B, C=C, D=D, init_state=h0)


def rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


# p1: the recurrent (scan) order and the quadratic (masked attention) order of
# the same semiseparable matrix agree.
@pytest.mark.parametrize("G", [1, 2, 4])
@pytest.mark.parametrize("with_init", [False, True])
def test_recurrent_equals_quadratic(G, with_init):
    rng = np.random.default_rng(100 + G)
    c = rand_case(rng, G=G, with_init=with_init)
    y_r, s_r = oracle.recurrent(**c)
    y_q, s_q = oracle.quadratic(**c)
    assert rel(y_q, y_r) < 1e-12
    assert rel(s_q, s_r) < 1e-12


# p2: the blocked (chunked) contraction is invariant to the chunk length,
# including chunk 1, a chunk longer than the sequence and a ragged last chunk.
@pytest.mark.parametrize("L,Q", [(64, 1), (64, 2), (64, 4), (64, 16), (64, 64), (64, 200),
                                 (50, 16), (37, 8), (1, 4)])
def test_recurrent_equals_chunked(L, Q):
    rng = np.random.default_rng(200 + L + Q)
    c = rand_case(rng, L=L, G=2)
    y_r, s_r = oracle.recurrent(**c)
    y_c, s_c = oracle.chunked(**c, chunk=Q)
    assert rel(y_c, y_r) < 1e-12
    assert rel(s_c, s_r) < 1e-12


# p3: A = 0 turns the layer into causal linear attention
#     y_i = sum_{j<=i} (C_i . B_j) dt_j x_j + C_i^T h0 + D x_i,
# written here as dense matrix products with a causal mask (numpy only).
def test_a_zero_is_causal_linear_attention():
    rng = np.random.default_rng(3)
    c = rand_case(rng, b=2, L=29, H=4, P=3, N=5, G=2)
    c["A"] = np.zeros(4)
    y, s = oracle.recurrent(**c)
    H, G = 4, 2
    for b in range(2):
        for h in range(H):
            g = h // (H // G)
            z = c["dt_raw"][b, :, h] + c["dt_bias"][h]
            dt = np.log1p(np.exp(z))
            Cg, Bg = c["C"][b, :, g, :], c["B"][b, :, g, :]
            xh = c["x"][b, :, h, :]
            h0 = c["init_state"][b, h]
            scores = np.tril(Cg @ Bg.T) * dt[None, :]
            expect = scores @ xh + Cg @ h0 + c["D"][h] * xh
            assert rel(y[b, :, h, :], expect) < 1e-12
            expect_state = h0 + Bg.T @ (dt[:, None] * xh)
            assert rel(s[b, h], expect_state) < 1e-12


# p4: dt -> 0 (softplus underflows to exactly 0): the state never moves, so
# y = C^T h0 + D x, y = D x exactly with a zero state, final_state = init_state.
@pytest.mark.parametrize("form", ["recurrent", "quadratic", "chunked"])
def test_dt_to_zero(form):
    rng = np.random.default_rng(4)
    c = rand_case(rng, b=1, L=20, H=2, P=3, N=4, G=1)
    c["dt_raw"] = np.full_like(c["dt_raw"], -1e4)
    c["dt_bias"] = np.zeros(2)
    fn = getattr(oracle, form)
    kw = {"chunk": 7} if form == "chunked" else {}
    y, s = fn(**c, **kw)
    expect = np.einsum("blgn,bhnp->blhp", c["C"], c["init_state"]) + c["D"][None, None, :, None] * c["x"]
    assert rel(y, expect) < 1e-13
    assert np.array_equal(s, c["init_state"])
    c0 = dict(c, init_state=None)
    y0, s0 = fn(**c0, **kw)
    assert np.array_equal(y0, c["D"][None, None, :, None] * c["x"])
    assert not np.any(s0)


# p5: prefill(L) == prefill(L1) followed by prefill(L - L1) from its final state.
@pytest.mark.parametrize("form", ["recurrent", "quadratic", "chunked"])
def test_split_handoff(form):
    rng = np.random.default_rng(5)
    c = rand_case(rng, L=40)
    fn = getattr(oracle, form)
    kw = {"chunk": 6} if form == "chunked" else {}
    y, s = fn(**c, **kw)
    L1 = 17
    first = {k: (v[:, :L1] if k in ("x", "dt_raw", "B", "C") else v) for k, v in c.items()}
    y1, s1 = fn(**first, **kw)
    second = {k: (v[:, L1:] if k in ("x", "dt_raw", "B", "C") else v) for k, v in c.items()}
    second["init_state"] = s1
    y2, s2 = fn(**second, **kw)
    assert rel(np.concatenate([y1, y2], axis=1), y) < 1e-12
    assert rel(s2, s) < 1e-12


# p6: scalar state (N = P = 1) with constant dt, A, B, x: the recurrence is a
# geometric series, h_T = dt b x (1 - q^T) / (1 - q), q = exp(dt A), and
# y_T = c h_T + D x (state AFTER the token-T update).
@pytest.mark.parametrize("form", ["recurrent", "quadratic", "chunked"])
def test_scalar_geometric_series(form):
    L, zr, bias, a, bv, xv, cv, dv = 50, 0.3, -0.7, -1.3, 0.8, -1.7, 0.45, 0.6
    dt = math.log1p(math.exp(zr + bias))
    q = math.exp(dt * a)
    case = dict(x=np.full((1, L, 1, 1), xv), dt_raw=np.full((1, L, 1), zr), dt_bias=np.array([bias]),
                A=np.array([a]), B=np.full((1, L, 1, 1), bv), C=np.full((1, L, 1, 1), cv),
                D=np.array([dv]), init_state=None)
    kw = {"chunk": 8} if form == "chunked" else {}
    y, s = getattr(oracle, form)(**case, **kw)
    for t in range(L):
        T = t + 1
        h_T = dt * bv * xv * (1 - q ** T) / (1 - q)
        assert abs(y[0, t, 0, 0] - (cv * h_T + dv * xv)) <= 1e-14 * max(1.0, abs(cv * h_T + dv * xv))
    h_L = dt * bv * xv * (1 - q ** L) / (1 - q)
    assert abs(s[0, 0, 0, 0] - h_L) <= 1e-14 * abs(h_L)


# p6b: impulse response with a varying dt: an input only at token 0 and a zero
# initial state decay by exp(A * sum_{k=1..t} dt_k) -- the cumulative decay
# includes token t itself but not token 0 (an off-by-one in the cumsum fails).
@pytest.mark.parametrize("form", ["recurrent", "quadratic", "chunked"])
def test_impulse_response_varying_dt(form):
    rng = np.random.default_rng(6)
    L = 33
    zr = rng.standard_normal(L)
    a, bv, xv, cv = -2.1, 1.3, 0.9, -0.7
    x = np.zeros((1, L, 1, 1))
    x[0, 0, 0, 0] = xv
    case = dict(x=x, dt_raw=zr.reshape(1, L, 1), dt_bias=np.array([0.0]), A=np.array([a]),
                B=np.full((1, L, 1, 1), bv), C=np.full((1, L, 1, 1), cv), D=np.array([0.0]), init_state=None)
    kw = {"chunk": 5} if form == "chunked" else {}
    y, _ = getattr(oracle, form)(**case, **kw)
    dt = np.log1p(np.exp(zr))
    for t in range(L):
        expect = cv * math.exp(a * float(np.sum(dt[1:t + 1]))) * dt[0] * bv * xv
        assert abs(y[0, t, 0, 0] - expect) <= 1e-13 * max(abs(expect), 1e-300)


# p7: linearity in x (for fixed dt, B, C) and in the initial state.
def test_linearity():
    rng = np.random.default_rng(7)
    c = rand_case(rng)
    x2 = rng.standard_normal(c["x"].shape)
    al, be = 0.7, -1.9
    y1, s1 = oracle.recurrent(**dict(c, init_state=None))
    y2, s2 = oracle.recurrent(**dict(c, x=x2, init_state=None))
    y3, s3 = oracle.recurrent(**dict(c, x=al * c["x"] + be * x2, init_state=None))
    assert rel(y3, al * y1 + be * y2) < 1e-12
    assert rel(s3, al * s1 + be * s2) < 1e-12
    h_a = c["init_state"]
    h_b = rng.standard_normal(h_a.shape)
    ya, sa = oracle.recurrent(**dict(c, init_state=h_a))
    yb, sb = oracle.recurrent(**dict(c, init_state=h_b))
    yab, sab = oracle.recurrent(**dict(c, init_state=h_a + h_b))
    # residual of the superposition, measured against the size of the outputs
    scale_y = max(np.max(np.abs(ya)), np.max(np.abs(yb)), np.max(np.abs(y1)))
    scale_s = max(np.max(np.abs(sa)), np.max(np.abs(sb)), np.max(np.abs(s1)))
    assert np.max(np.abs((yab - y1) - (ya - y1) - (yb - y1))) < 1e-13 * scale_y
    assert np.max(np.abs((sab - s1) - (sa - s1) - (sb - s1))) < 1e-13 * scale_s
    # and the initial-state contribution is not negligible in this case
    assert np.max(np.abs(ya - y1)) > 1e-3 * scale_y


# p7b: G = H with B, C replicated per head equals G = 1.
def test_groups_replicated():
    rng = np.random.default_rng(8)
    c = rand_case(rng, G=1)
    y1, s1 = oracle.recurrent(**c)
    rep = dict(c, B=np.repeat(c["B"], 4, axis=2), C=np.repeat(c["C"], 4, axis=2))
    y4, s4 = oracle.recurrent(**rep)
    assert np.array_equal(y1, y4) and np.array_equal(s1, s4)


# p7c: head h reads group h // (H/G): each head equals a one-head run on its group.
def test_group_mapping():
    rng = np.random.default_rng(9)
    H, G = 6, 3
    c = rand_case(rng, H=H, G=G)
    y, s = oracle.recurrent(**c)
    for h in range(H):
        g = h // (H // G)
        one = dict(x=c["x"][:, :, h:h + 1], dt_raw=c["dt_raw"][:, :, h:h + 1], dt_bias=c["dt_bias"][h:h + 1],
                   A=c["A"][h:h + 1], B=c["B"][:, :, g:g + 1], C=c["C"][:, :, g:g + 1], D=c["D"][h:h + 1],
                   init_state=c["init_state"][:, h:h + 1])
        yh, sh = oracle.recurrent(**one)
        assert np.array_equal(yh[:, :, 0], y[:, :, h]) and np.array_equal(sh[:, 0], s[:, h])


# decode: one step equals the recurrence over one token from the same state.
def test_decode_step_equals_recurrent_one_token():
    rng = np.random.default_rng(10)
    c = rand_case(rng, b=3, L=1, H=4, P=5, N=6, G=2)
    y_r, s_r = oracle.recurrent(**c)
    st = c["init_state"].copy()
    y_d = oracle.decode_step(st, c["x"][:, 0], c["dt_raw"][:, 0], c["dt_bias"], c["A"], c["B"][:, 0],
                             c["C"][:, 0], c["D"])
    assert rel(y_d, y_r[:, 0]) < 1e-14
    assert rel(st, s_r) < 1e-14


def test_decode_steps_equal_prefill():
    rng = np.random.default_rng(11)
    c = rand_case(rng, b=2, L=12, H=4, P=3, N=5, G=2)
    y_r, s_r = oracle.recurrent(**c)
    st = c["init_state"].copy()
    for t in range(12):
        y_d = oracle.decode_step(st, c["x"][:, t], c["dt_raw"][:, t], c["dt_bias"], c["A"], c["B"][:, t],
                                 c["C"][:, t], c["D"])
        assert rel(y_d, y_r[:, t]) < 1e-13
    assert rel(st, s_r) < 1e-13


# bf16 state storage: the stored state is the bf16 rounding of the float64
# update; y comes from the unrounded update.
def test_decode_bf16_state_rounding():
    rng = np.random.default_rng(12)
    c = rand_case(rng, b=2, L=1, H=4, P=3, N=5, G=2)
    st_exact = c["init_state"].copy()
    y_exact = oracle.decode_step(st_exact, c["x"][:, 0], c["dt_raw"][:, 0], c["dt_bias"], c["A"],
                                 c["B"][:, 0], c["C"][:, 0], c["D"])
    st = c["init_state"].copy()
    y = oracle.decode_step(st, c["x"][:, 0], c["dt_raw"][:, 0], c["dt_bias"], c["A"], c["B"][:, 0],
                           c["C"][:, 0], c["D"], round_state_bf16=True)
    assert np.array_equal(y, y_exact)
    assert np.array_equal(st, oracle.round_bf16(st_exact))
    assert not np.array_equal(st, st_exact)


def test_round_bf16_against_torch_and_ties():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(13)
    v = np.concatenate([rng.standard_normal(2000) * 10.0 ** rng.integers(-30, 30, 2000),
                        [1.0, -1.0, 3.0e38, 1e-40, 0.0]]).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(oracle.round_bf16(v.astype(np.float64)), ref)
    # ties go to the even neighbour: bf16 spacing at 1.0 is 2^-7
    assert oracle.round_bf16(1 + 2.0 ** -8) == 1.0
    assert oracle.round_bf16(1 + 2.0 ** -7 + 2.0 ** -8) == 1 + 2.0 ** -6
    # the generator's bf16 rounding agrees with the oracle's on fp32-representable values
    assert np.array_equal(I.to_f64(I.to_storage(v, I.BF16)), ref)


def test_softplus_values():
    assert abs(oracle.softplus(0.0) - math.log(2.0)) < 1e-16
    assert oracle.softplus(-1e4) == 0.0
    assert oracle.softplus(800.0) == 800.0
    for z in (-30.0, -3.0, -0.5, 0.5, 3.0, 30.0):
        assert abs(oracle.softplus(z) - math.log1p(math.exp(z))) <= 1e-15 * max(1.0, abs(z))


def test_generator_distributions():
    # the input recipe: dt_bias = log(expm1(U[1e-3, 1e-1])) => softplus(dt_bias) in [1e-3, 1e-1]
    p = I.draw_head_params(4096, seed=0)
    sp = np.log1p(np.exp(p["dt_bias"].astype(np.float64)))
    assert sp.min() >= 1e-3 * (1 - 1e-6) and sp.max() <= 1e-1 * (1 + 1e-6)
    assert -16.0 <= p["A"].min() and p["A"].max() <= -1.0
    s = I.draw_decode_state(0, 64, 64, 128, seed=3, dtype=I.F32)
    assert abs(float(s.std()) - 0.1) < 2e-3
    # slices regenerate independently
    a = I.prefill_inputs(3, 16, 2, 8, 4, 1, 5, I.BF16)
    b = I.prefill_inputs(3, 16, 2, 8, 4, 1, 5, I.BF16, batches=[2])
    assert np.array_equal(a["x"][2], b["x"][0])


def test_invalid_arguments_raise():
    rng = np.random.default_rng(14)
    c = rand_case(rng, H=4, G=2)
    bad = dict(c, B=c["B"][:, :, :1].repeat(3, axis=2), C=c["C"][:, :, :1].repeat(3, axis=2))
    with pytest.raises(ValueError):
        oracle.recurrent(**bad)  # H % G != 0


# regression: the oracle still reproduces the committed fixture (written by
# tests/golden/make_golden.py, which calls only the oracle)
def test_golden_regression():
    import json
    import os
    import tests.golden.make_golden as mg
    with open(os.path.join(os.path.dirname(mg.__file__), "oracle_tiny.json")) as f:
        gold = json.load(f)
    inp, h0 = mg.case()
    y, fs = oracle.recurrent(inp["x"], inp["dt_raw"], inp["dt_bias"], inp["A"], inp["B"], inp["C"], inp["D"],
                             init_state=h0)
    assert rel(y.ravel(), np.array(gold["y"])) < 1e-14
    assert rel(fs.ravel(), np.array(gold["final_state"])) < 1e-14


# MIMO decode (rank R): pinned by compositions of the (pinned) single-input step.
def _mimo_case(rng, b=2, H=4, P=3, N=5, G=2, R=3):
    return dict(state=rng.standard_normal((b, H, N, P)), x=rng.standard_normal((b, H, R, P)),
                dt_raw=rng.standard_normal((b, H)), dt_bias=np.log(np.expm1(rng.uniform(1e-2, 0.5, H))),
                A=-rng.uniform(0.5, 4.0, H), B=rng.standard_normal((b, G, R, N)),
                C=rng.standard_normal((b, G, R, N)), D=rng.standard_normal(H))


def test_mimo_rank1_is_the_decode_step():
    c = _mimo_case(np.random.default_rng(31), R=1)
    st1, st2 = c["state"].copy(), c["state"].copy()
    y1 = oracle.decode_step_mimo(st1, c["x"], c["dt_raw"], c["dt_bias"], c["A"], c["B"], c["C"], c["D"])
    y2 = oracle.decode_step(st2, c["x"][:, :, 0], c["dt_raw"], c["dt_bias"], c["A"], c["B"][:, :, 0],
                            c["C"][:, :, 0], c["D"])
    assert rel(y1[:, :, 0], y2) < 1e-14 and rel(st1, st2) < 1e-14


@pytest.mark.parametrize("R", [2, 4])
def test_mimo_step_is_a_chain_of_single_input_steps(R):
    """h <- exp(dt A) h + dt sum_r B_r x_r^T is one single-input step with input 0
    followed by R-1 single-input steps with A = 0 (no decay) and the same dt; output
    r is the last output of such a chain that ends with input r and reads C_r."""
    c = _mimo_case(np.random.default_rng(40 + R), R=R)
    st = c["state"].copy()
    y = oracle.decode_step_mimo(st, c["x"], c["dt_raw"], c["dt_bias"], c["A"], c["B"], c["C"], c["D"])
    zeroA = np.zeros_like(c["A"])
    for r_last in range(R):
        order = [r for r in range(R) if r != r_last] + [r_last]
        chain = c["state"].copy()
        for i, r in enumerate(order):
            yc = oracle.decode_step(chain, c["x"][:, :, r], c["dt_raw"], c["dt_bias"], c["A"] if i == 0 else zeroA,
                                    c["B"][:, :, r], c["C"][:, :, r_last], c["D"])
        assert rel(chain, st) < 1e-13
        assert rel(yc, y[:, :, r_last]) < 1e-13


def test_mimo_bf16_state_rounding():
    c = _mimo_case(np.random.default_rng(52), R=2)
    exact, rounded = c["state"].copy(), c["state"].copy()
    y1 = oracle.decode_step_mimo(exact, c["x"], c["dt_raw"], c["dt_bias"], c["A"], c["B"], c["C"], c["D"])
    y2 = oracle.decode_step_mimo(rounded, c["x"], c["dt_raw"], c["dt_bias"], c["A"], c["B"], c["C"], c["D"],
                                 round_state_bf16=True)
    assert np.array_equal(y1, y2)
    assert np.array_equal(rounded, oracle.round_bf16(exact))


# p-mimo-seq: the MIMO sequence oracle is the (separately pinned) MIMO decode
# step applied token by token, and at rank 1 the SISO recurrence
@pytest.mark.parametrize("R", [1, 3])
def test_mimo_sequence_is_a_chain_of_mimo_steps(R):
    rng = np.random.default_rng(70 + R)
    b, L, H, P, N, G = 2, 11, 4, 3, 5, 2
    x = rng.standard_normal((b, L, H, R, P))
    dt_raw = rng.standard_normal((b, L, H))
    dt_bias = rng.uniform(-1, 0.5, H)
    A = -rng.uniform(0.5, 3.0, H)
    B = rng.standard_normal((b, L, G, R, N))
    C = rng.standard_normal((b, L, G, R, N))
    D = rng.standard_normal(H)
    h0 = rng.standard_normal((b, H, N, P))
    y, fs = oracle.mimo_recurrent(x, dt_raw, dt_bias, A, B, C, D, h0)
    st = h0.copy()
    for t in range(L):
        yt = oracle.decode_step_mimo(st, x[:, t], dt_raw[:, t], dt_bias, A, B[:, t], C[:, t], D)
        assert rel(y[:, t], yt) < 1e-13
    assert rel(fs, st) < 1e-13
    if R == 1:
        y1, f1 = oracle.recurrent(x[:, :, :, 0], dt_raw, dt_bias, A, B[:, :, :, 0], C[:, :, :, 0], D, h0)
        assert rel(y[:, :, :, 0], y1) < 1e-13 and rel(fs, f1) < 1e-13
