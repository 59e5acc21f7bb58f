"""GPU parity of ssd_chunk_scan_fwd against the float64 oracle (small and
medium shapes: several chunks, ragged tails, both kernel paths, all dtype
combinations, initial states, cross-path invariants)."""
import numpy as np
import pytest

from mamba_ssd_scan_chunked_b200 import inputs as I
from mamba_ssd_scan_chunked_b200 import ssd
from tests.gpu_util import (TOL_BF16, TOL_F32, bf16_excess_metric, gpu_prefill, metric, oracle_prefill,
                            random_state, to_dev, to_host64, torch)

pytestmark = pytest.mark.gpu


def shape_inputs(b, L, H, P, N, G, dtype, seed):
    return I.prefill_inputs(b, L, H, P, N, G, seed, dtype)


def path_of(inp, chunk):
    t = torch()
    x = to_dev(inp["x"][:, :1])
    Bm = to_dev(inp["B"][:, :1])
    return ssd.ssd_chunk_scan_path(ssd.prefill_desc(x, Bm, chunk))


# (b, L, H, P, N, G, chunk, dtype) -- L is not a multiple of the chunk in most cases
CASES = [
    (2, 300, 4, 64, 16, 2, 64, I.F32),      # fp32, CUDA cores, ragged tail
    (1, 256, 4, 64, 16, 1, 64, I.F32),
    (2, 200, 3, 32, 24, 3, 32, I.F32),      # odd head count, G = H
    (1, 130, 2, 64, 64, 1, 16, I.F32),
    (2, 600, 4, 64, 128, 2, 256, I.BF16),   # bf16, tensor cores: 3 chunks, last has 88 tokens
    (2, 384, 4, 64, 128, 1, 128, I.BF16),   # tensor cores, chunk 128
    (1, 1000, 6, 64, 128, 3, 256, I.BF16),  # tensor cores, 4 chunks, ragged 232-token tail
    (2, 333, 4, 64, 64, 2, 64, I.BF16),     # bf16 on CUDA cores
    (1, 257, 2, 128, 256, 1, 128, I.BF16),
    (1, 3918, 100, 64, 128, 4, 128, I.BF16),  # tensor cores, runs of 4 chunks, the last run 3 chunks
    (2, 600, 4, 64, 64, 2, 256, I.BF16),    # dstate 64 on tensor cores (zero-padded B), runs
    (1, 2100, 90, 64, 64, 3, 256, I.BF16),  # dstate 64, 90 sequences cut into runs of 1 chunk
    (1, 1000, 6, 64, 256, 3, 128, I.BF16),  # dstate 256: one pipeline per SM, two state halves, runs
    (2, 1500, 80, 64, 256, 8, 256, I.BF16), # dstate 256, whole sequences, 160 items on 148 CTAs
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "b{}_L{}_H{}_P{}_N{}_G{}_Q{}_{}".format(*c))
@pytest.mark.parametrize("with_init", [False, True])
def test_prefill_matches_oracle(case, with_init):
    b, L, H, P, N, G, Q, dt = case
    inp = shape_inputs(b, L, H, P, N, G, dt, seed=11 + L)
    h0 = random_state((b, H, N, P), 5 + L, I.F32) if with_init else None
    y, fs = gpu_prefill(inp, Q, h0)
    y_ref, fs_ref = oracle_prefill(inp, h0)
    tol = TOL_F32 if dt == I.F32 else TOL_BF16
    assert metric(y, y_ref) <= tol
    assert metric(fs, fs_ref) <= tol


# (b, L, H, G, chunk) of the head-pair kernel: dstate 128, an even number of heads
# per group, >= 148 sequences
PAIR_CASES = [
    (1, 300, 148, 2, 256),    # 74 items, 3 blocks, ragged 44-token tail
    (2, 520, 80, 4, 128),     # 80 items, chunk 128, an 8-token tail block
    (1, 260, 400, 8, 128),    # 200 items on at most 148 CTAs: some CTAs take two
]


@pytest.mark.parametrize("case", PAIR_CASES, ids=lambda c: "b{}_L{}_H{}_G{}_Q{}".format(*c))
@pytest.mark.parametrize("with_init", [False, True])
def test_head_pair_path_matches_oracle(case, with_init):
    b, L, H, G, Q = case
    inp = shape_inputs(b, L, H, 64, 128, G, I.BF16, seed=41 + L)
    assert path_of(inp, Q) == 2
    h0 = random_state((b, H, 128, 64), 43 + L, I.F32) if with_init else None
    y, fs = gpu_prefill(inp, Q, h0)
    y_ref, fs_ref = oracle_prefill(inp, h0)
    # same arithmetic as the single-head kernel: far inside the 2e-2 bound
    assert metric(y, y_ref) < 2e-3
    assert metric(fs, fs_ref) < 2e-3


def test_head_pair_bf16_outputs_and_states():
    inp = shape_inputs(2, 384, 80, 64, 128, 2, I.BF16, 23)
    h0 = random_state((2, 80, 128, 64), 24, I.BF16)
    y, fs = gpu_prefill(inp, 256, h0, y_dtype="bf16", state_dtype="bf16")
    y_ref, fs_ref = oracle_prefill(inp, h0)
    assert bf16_excess_metric(y, y_ref) <= TOL_BF16
    assert bf16_excess_metric(fs, fs_ref) <= TOL_BF16


def test_head_pair_positive_decay_exponent():
    """A > 0 on some heads: the log-decay grows, and blocks of those pairs take the
    per-element decay factors instead of the split ones."""
    inp = shape_inputs(1, 400, 148, 64, 128, 2, I.BF16, 25)
    A = inp["A"].copy()
    A[[3, 4, 77]] = np.float32(0.02)
    inp["A"] = A
    y, fs = gpu_prefill(inp, 256)
    y_ref, fs_ref = oracle_prefill(inp)
    assert metric(y, y_ref) < 2e-3
    assert metric(fs, fs_ref) < 2e-3


@pytest.mark.parametrize("N", [64, 128, 256])
def test_tensor_core_path_is_taken_for_bf16_headdim64(N):
    inp = shape_inputs(1, 256, 2, 64, N, 1, I.BF16, 3)
    assert path_of(inp, 256) == 0
    assert path_of(inp, 128) == 0
    assert path_of(inp, 64) == 1                      # chunk 64: CUDA cores
    inp32 = shape_inputs(1, 256, 2, 64, N, 1, I.F32, 3)
    assert path_of(inp32, 256) == 1
    assert path_of(shape_inputs(1, 256, 2, 64, 32, 1, I.BF16, 3), 256) == 1   # dstate 32: CUDA cores


def test_tensor_core_error_budget_is_far_inside_the_bound():
    # the hi/lo split keeps the tensor-core path ~100x inside the 2e-2 bound
    inp = shape_inputs(2, 1024, 8, 64, 128, 2, I.BF16, 77)
    y, fs = gpu_prefill(inp, 256)
    y_ref, fs_ref = oracle_prefill(inp)
    assert metric(y, y_ref) < 2e-3
    assert metric(fs, fs_ref) < 2e-3


@pytest.mark.parametrize("Q", [256, 64])
def test_bf16_outputs(Q):
    """y and final_state stored in bf16: the error beyond the output's own rounding stays in bounds."""
    N = 128 if Q == 256 else 64
    inp = shape_inputs(2, 512, 4, 64, N, 2, I.BF16, 21)
    h0 = random_state((2, 4, N, 64), 22, I.BF16)
    y, fs = gpu_prefill(inp, Q, h0, y_dtype="bf16", state_dtype="bf16")
    y_ref, fs_ref = oracle_prefill(inp, h0)
    assert bf16_excess_metric(y, y_ref) <= TOL_BF16
    assert bf16_excess_metric(fs, fs_ref) <= TOL_BF16


def test_zero_init_buffer_equals_null_init():
    inp = shape_inputs(1, 512, 4, 64, 128, 2, I.BF16, 31)
    y0, f0 = gpu_prefill(inp, 256)
    z = np.zeros((1, 4, 128, 64), np.float32)
    y1, f1 = gpu_prefill(inp, 256, z)
    assert np.array_equal(y0, y1) and np.array_equal(f0, f1)


@pytest.mark.parametrize("dt", [I.F32, I.BF16])
def test_split_prefill_handoff(dt):
    """prefill(L) == prefill(L1) then prefill(L - L1) from its final state."""
    b, L, H, P, N, G, Q = 2, 768, 4, 64, 128, 2, 256
    inp = shape_inputs(b, L, H, P, N, G, dt, 41)
    y, fs = gpu_prefill(inp, Q)
    L1 = 512
    first = {k: (v[:, :L1] if k in ("x", "dt_raw", "B", "C") else v) for k, v in inp.items()}
    second = {k: (np.ascontiguousarray(v[:, L1:]) if k in ("x", "dt_raw", "B", "C") else v) for k, v in inp.items()}
    first = {k: np.ascontiguousarray(v) for k, v in first.items()}
    y1, f1 = gpu_prefill(first, Q)
    y2, f2 = gpu_prefill(second, Q, f1.astype(np.float32))
    tol = TOL_F32 if dt == I.F32 else TOL_BF16
    assert metric(np.concatenate([y1, y2], axis=1), y) <= tol
    assert metric(f2, fs) <= tol


def test_empty_sequence_copies_init_state():
    t = torch()
    inp = shape_inputs(2, 0, 4, 64, 128, 2, I.BF16, 51)
    h0 = random_state((2, 4, 128, 64), 52, I.F32)
    y, fs = gpu_prefill(inp, 256, h0)
    assert y.shape == (2, 0, 4, 64)
    assert np.array_equal(fs, I.to_f64(h0))
    _, fz = gpu_prefill(inp, 256, None)
    assert not np.any(fz)


def test_device_error_word_clear_after_runs():
    st, detail = ssd.ssd_get_device_error(0)
    assert st == 0 and detail == 0
