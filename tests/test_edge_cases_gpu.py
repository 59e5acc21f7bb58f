"""GPU parity on the method's degenerate and extreme cases, on every prefill
kernel path and on the decode step:

- A = 0: no decay; the layer is causal linear attention, y_i = sum_{j<=i}
  (C_i . B_j) dt_j x_j + C_i h0 + D x_i ("Mamba-2 vs Transformers / SSD",
  section "Mamba-2 and the SSD paper: what changed in practice": the SSM as a
  masked, attention-like contraction);
- dt -> 0 (dt_raw = -1e4): the step neither decays nor feeds the state, so y =
  C h0 + D x and the final state is the initial one ("Mamba3", section "New
  discretisation scheme": dt scales both the decay exponent and the input);
- softplus above its switch (dt_raw = +30, z > 20): dt = z;
- decays that underflow inside a block (A = -16, dt ~ 5: a = -80 per token).

Each is compared with the float64 oracle on the same stored values; A = 0 and
dt -> 0 also against their closed forms written out here."""
import numpy as np
import pytest

import oracle
from mamba_ssd_scan_chunked_b200 import inputs as I
from mamba_ssd_scan_chunked_b200 import ssd
from tests.gpu_util import (TOL_BF16, TOL_F32, bf16_state_metric, gpu_prefill, metric, oracle_prefill,
                            random_state, to_dev, to_host64, torch)

pytestmark = pytest.mark.gpu

# (b, L, H, P, N, G, chunk, dtype, expected path)
PATHS = {
    "tensor_cores": (2, 600, 4, 64, 128, 2, 256, I.BF16, 0),         # sequences cut into runs
    "tensor_cores_head_pairs": (1, 300, 148, 64, 128, 2, 256, I.BF16, 2),
    "tensor_cores_dstate64": (2, 300, 4, 64, 64, 2, 128, I.BF16, 0),
    "cuda_cores_fp32": (2, 300, 4, 64, 16, 2, 64, I.F32, 1),
}
CASES = ["a_zero", "dt_to_zero", "softplus_above_switch", "underflowing_decay"]


def edge_inputs(case, b, L, H, P, N, G, dtype, seed):
    inp = I.prefill_inputs(b, L, H, P, N, G, seed, dtype)
    rng = np.random.default_rng(seed + 1000)
    dt_raw = I.to_f64(inp["dt_raw"])
    if case == "a_zero":
        inp["A"] = np.zeros(H, np.float32)
    elif case == "dt_to_zero":
        inp["dt_raw"] = I.to_storage(np.full(dt_raw.shape, -1e4), dtype)
    elif case == "softplus_above_switch":
        hot = rng.random(dt_raw.shape) < 0.15
        inp["dt_raw"] = I.to_storage(np.where(hot, 30.0, dt_raw), dtype)
    elif case == "underflowing_decay":
        hot = rng.random(dt_raw.shape) < 0.5
        inp["dt_raw"] = I.to_storage(np.where(hot, 5.0, dt_raw), dtype)
        inp["dt_bias"] = np.zeros(H, np.float32)
        inp["A"] = np.full(H, -16.0, np.float32)
    return inp


def causal_linear_attention(inp, h0):
    """y for A = 0, written out as masked matmuls per (batch, head)."""
    f = {k: I.to_f64(v) for k, v in inp.items()}
    x, B, C = f["x"], f["B"], f["C"]
    b, L, H, P = x.shape
    G = B.shape[2]
    z = f["dt_raw"] + f["dt_bias"][None, None, :]
    dt = np.array([[[oracle.softplus(v) for v in row] for row in bat] for bat in z])
    mask = np.tril(np.ones((L, L)))
    y = np.empty_like(x)
    for bi in range(b):
        for h in range(H):
            g = h // (H // G)
            S = (C[bi, :, g] @ B[bi, :, g].T) * mask
            y[bi, :, h] = S @ (dt[bi, :, h, None] * x[bi, :, h]) + f["D"][h] * x[bi, :, h]
            if h0 is not None:
                y[bi, :, h] += C[bi, :, g] @ h0[bi, h]
    return y


def path_of(inp, chunk):
    x = to_dev(inp["x"][:, :1])
    Bm = to_dev(inp["B"][:, :1])
    return ssd.ssd_chunk_scan_path(ssd.prefill_desc(x, Bm, chunk))


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("path", list(PATHS))
def test_prefill_edge_case(path, case):
    b, L, H, P, N, G, Q, dtype, want = PATHS[path]
    inp = edge_inputs(case, b, L, H, P, N, G, dtype, seed=61)
    assert path_of(inp, Q) == want
    h0 = random_state((b, H, N, P), 62, I.F32)
    y, fs = gpu_prefill(inp, Q, h0)
    y_ref, fs_ref = oracle_prefill(inp, h0)
    tol = TOL_F32 if dtype == I.F32 else TOL_BF16
    assert np.all(np.isfinite(y)) and np.all(np.isfinite(fs))
    assert metric(y, y_ref) <= tol
    assert metric(fs, fs_ref) <= tol
    if case == "a_zero":
        assert metric(y, causal_linear_attention(inp, I.to_f64(h0))) <= tol
    if case == "dt_to_zero":
        f = {k: I.to_f64(v) for k, v in inp.items()}
        g_of_h = np.arange(H) // (H // G)
        closed = np.einsum("blhn,bhnp->blhp", f["C"][:, :, g_of_h], I.to_f64(h0)) + f["D"][None, None, :, None] * f["x"]
        assert metric(y, closed) <= tol
        # no input and a decay of exactly 1: the state is returned unchanged
        assert np.array_equal(fs, I.to_f64(h0))


def run_decode(state0, steps, params):
    t = torch()
    st = to_dev(state0)
    prm = {k: to_dev(v) for k, v in params.items()}
    ys = []
    for s in steps:
        d = {k: to_dev(v) for k, v in s.items()}
        ys.append(to_host64(ssd.state_update(st, d["x"], d["dt_raw"], prm["dt_bias"], prm["A"], d["B"], d["C"],
                                             prm["D"], y_dtype=t.float32)))
    t.cuda.synchronize()
    return ys, to_host64(st)


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("state_dtype", [I.F32, I.BF16])
def test_decode_edge_case(case, state_dtype):
    b, H, P, N, G, T = 4, 8, 64, 128, 2, 5
    params = I.draw_head_params(H, seed=71)
    st0 = np.stack([I.draw_decode_state(i, H, P, N, seed=72, dtype=state_dtype) for i in range(b)])
    rng = np.random.default_rng(73)
    steps = []
    for t in range(T):
        s = I.draw_decode_step(t, b, H, P, N, G, seed=74, dtype=I.BF16)
        dt_raw = I.to_f64(s["dt_raw"])
        if case == "dt_to_zero":
            s["dt_raw"] = I.to_storage(np.full(dt_raw.shape, -1e4), I.BF16)
        elif case == "softplus_above_switch":
            s["dt_raw"] = I.to_storage(np.where(rng.random(dt_raw.shape) < 0.5, 30.0, dt_raw), I.BF16)
        elif case == "underflowing_decay":
            s["dt_raw"] = I.to_storage(np.where(rng.random(dt_raw.shape) < 0.5, 5.0, dt_raw), I.BF16)
        steps.append(s)
    if case == "a_zero":
        params["A"] = np.zeros(H, np.float32)
    elif case == "underflowing_decay":
        params["A"] = np.full(H, -16.0, np.float32)
        params["dt_bias"] = np.zeros(H, np.float32)
    ys, s_gpu = run_decode(st0, steps, params)
    st = I.to_f64(st0).copy()
    f = {k: I.to_f64(v) for k, v in params.items()}
    for y, s in zip(ys, steps):
        g = {k: I.to_f64(v) for k, v in s.items()}
        y_ref = oracle.decode_step(st, g["x"], g["dt_raw"], f["dt_bias"], f["A"], g["B"], g["C"], f["D"],
                                   round_state_bf16=(state_dtype == I.BF16))
        assert metric(y, y_ref) <= TOL_BF16
    state_metric = bf16_state_metric if state_dtype == I.BF16 else metric
    assert state_metric(s_gpu, st) <= TOL_BF16
    if case == "dt_to_zero":
        assert np.array_equal(s_gpu, I.to_f64(st0))
