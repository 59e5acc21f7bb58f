"""GPU parity of ssd_chunk_scan_bwd (the backward pass of the chunked scan)
against the float64 oracle's reverse-mode gradients of the sequential
recurrence, element by element, on the same seeded inputs.

The oracle gets the stored (bf16 or fp32) values exactly; every gradient is
returned in fp32 and compared with max|err| / rms(oracle) against the
tolerance of its input dtype (bf16 gradient outputs are checked beyond their
own rounding, in a test of their own).  Shapes span several chunks with a ragged last chunk, every dstate the
tensor-core path covers, the CUDA-core (fp32) path, sequences long enough to
be cut into runs, and the degenerate cases (no initial state, no final-state
gradient, empty sequence, empty batch)."""
import numpy as np
import pytest

import oracle
from mamba_ssd_scan_chunked_b200 import inputs as I
from mamba_ssd_scan_chunked_b200 import ssd
from tests.gpu_util import TOL_BF16, TOL_F32, bf16_excess_metric, metric, to_dev, to_host64, torch

pytestmark = pytest.mark.gpu

GRADS = ("dx", "ddt_raw", "dB", "dC", "dA", "ddt_bias", "dD", "dinit_state")


def make_case(b, L, H, P, N, G, io, state, seed, with_init, with_dfinal):
    inp = I.prefill_inputs(b, L, H, P, N, G, seed, io)
    if with_init:
        inp["init_state"] = np.stack([I.draw_decode_state(i, H, P, N, seed=seed + 1, dtype=state) for i in range(b)])
    seeds = I.draw_output_grads(b, L, H, P, N, seed, io, state)
    inp["dy"] = seeds["dy"]
    if with_dfinal:
        inp["dfinal"] = seeds["dfinal"]
    return inp


def run_both(inp, Q, grad_dtype="f32"):
    t = torch()
    if grad_dtype == "f32":
        grad_dtype = t.float32
    dev = {k: to_dev(v) for k, v in inp.items()}
    got = ssd.chunk_scan_bwd(dev["x"], dev["dt_raw"], dev["dt_bias"], dev["A"], dev["B"], dev["C"], dev["D"], Q,
                             dev["dy"], dev.get("init_state"), dev.get("dfinal"), grad_dtype=grad_dtype)
    t.cuda.synchronize()
    assert ssd.ssd_get_device_error(0)[0] == 0
    f = {k: I.to_f64(v) for k, v in inp.items()}
    ref = oracle.backward(f["x"], f["dt_raw"], f["dt_bias"], f["A"], f["B"], f["C"], f["D"], f.get("init_state"),
                          f["dy"], f.get("dfinal"))
    return {k: to_host64(v) for k, v in got.items() if v is not None}, ref


def worst(got, ref, skip=()):
    return {k: metric(got[k], ref[k]) for k in GRADS if k not in skip}


# Every gradient, d dt_raw, d dt_bias and dA included, is held to the flat
# bound of its input dtype at every sequence length: the fp32 path forms the
# log-decay gradient inside each block of the sequence from the block's own
# terms, the state entering the block and the adjoint leaving it, so its
# rounding error does not grow with the sequence.


def tolerances(io, L):
    base = TOL_BF16 if io == I.BF16 else TOL_F32
    return {k: base for k in GRADS}


@pytest.mark.parametrize("b,L,H,P,N,G,Q,io,with_init,with_dfinal", [
    (2, 300, 4, 64, 128, 2, 128, I.BF16, True, True),     # tensor cores, 3 chunks, ragged tail
    (2, 600, 2, 64, 64, 1, 256, I.BF16, False, False),    # dstate 64, no states
    (1, 260, 2, 64, 256, 2, 128, I.BF16, True, False),    # dstate 256 (4 column slices)
    (2, 200, 3, 32, 16, 3, 64, I.F32, True, True),        # CUDA-core path, fp32
    (1, 130, 2, 48, 24, 1, 32, I.F32, False, True),       # CUDA-core path, odd sizes
    (1, 1000, 2, 64, 128, 2, 256, I.F32, True, True),     # fp32, 32 blocks of 32 tokens, ragged tail
    (1, 70, 2, 256, 256, 1, 64, I.F32, True, True),       # fp32, largest head and state (16-token blocks)
])
def test_backward_matches_oracle(b, L, H, P, N, G, Q, io, with_init, with_dfinal):
    inp = make_case(b, L, H, P, N, G, io, I.F32, 11, with_init, with_dfinal)
    got, ref = run_both(inp, Q)
    tol = tolerances(io, L)
    errs = worst(got, ref)
    assert all(errs[k] <= tol[k] for k in GRADS), errs


def test_backward_long_sequences_cut_into_runs():
    """Two heads of 4096 tokens: the scans cut each sequence into runs with
    state hand-offs between them (forward and reversed in time)."""
    inp = make_case(1, 4096, 2, 64, 128, 1, I.BF16, I.F32, 12, True, True)
    got, ref = run_both(inp, 256)
    errs = worst(got, ref)
    assert max(errs.values()) <= TOL_BF16, errs


def test_backward_bf16_gradients_and_state():
    """bf16 gradient outputs and a bf16 state dtype (init, dfinal, dinit)."""
    inp = make_case(2, 256, 4, 64, 128, 1, I.BF16, I.BF16, 13, True, True)
    got, ref = run_both(inp, 128, grad_dtype=torch().bfloat16)
    for k in ("dx", "ddt_raw", "dB", "dC", "dinit_state"):
        assert bf16_excess_metric(got[k], ref[k]) <= TOL_BF16, k
    for k in ("dA", "ddt_bias", "dD"):
        assert metric(got[k], ref[k]) <= TOL_BF16, k


@pytest.mark.parametrize("io", [I.BF16, I.F32])
def test_backward_is_deterministic(io):
    t = torch()
    inp = make_case(2, 300, 4, 64, 128, 2, io, I.F32, 14, True, True)
    dev = {k: to_dev(v) for k, v in inp.items()}
    outs = [ssd.chunk_scan_bwd(dev["x"], dev["dt_raw"], dev["dt_bias"], dev["A"], dev["B"], dev["C"], dev["D"], 128,
                               dev["dy"], dev["init_state"], dev["dfinal"]) for _ in range(2)]
    t.cuda.synchronize()
    for k in GRADS:
        assert t.equal(outs[0][k], outs[1][k]), k


def test_backward_empty_sequence_and_batch():
    t = torch()
    H, P, N = 2, 64, 64
    dfinal = t.randn(2, H, N, P, device="cuda")
    x = t.empty(2, 0, H, P, device="cuda", dtype=t.bfloat16)
    B = t.empty(2, 0, 1, N, device="cuda", dtype=t.bfloat16)
    prm = {k: to_dev(v) for k, v in I.draw_head_params(H, seed=3).items()}
    out = ssd.chunk_scan_bwd(x, t.empty(2, 0, H, device="cuda", dtype=t.bfloat16), prm["dt_bias"], prm["A"], B, B,
                             prm["D"], 128, x, None, dfinal)
    t.cuda.synchronize()
    assert t.equal(out["dinit_state"], dfinal)
    for k in ("dA", "ddt_bias", "dD"):
        assert not t.any(out[k]), k
    x0 = t.empty(0, 5, H, P, device="cuda", dtype=t.bfloat16)
    B0 = t.empty(0, 5, 1, N, device="cuda", dtype=t.bfloat16)
    out = ssd.chunk_scan_bwd(x0, t.empty(0, 5, H, device="cuda", dtype=t.bfloat16), prm["dt_bias"], prm["A"], B0,
                             B0, prm["D"], 128, x0)
    t.cuda.synchronize()
    assert not t.any(out["dA"])
