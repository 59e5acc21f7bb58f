"""GPU parity of ssd_chunk_scan_fwd_varlen (left-padded variable-length
batches): every sequence, padded or not, must give the oracle's result for its
unpadded tokens alone, started from its initial state."""
import numpy as np
import pytest

import oracle
from mamba_ssd_scan_chunked_b200 import inputs as I
from mamba_ssd_scan_chunked_b200 import ssd
from tests.gpu_util import TOL_BF16, TOL_F32, metric, random_state, to_dev, to_host64, torch

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("b,L,H,P,N,G,Q,dt,pads", [
    (4, 600, 4, 64, 128, 2, 256, I.BF16, [0, 37, 300, 599]),     # tensor cores: pads inside, across, to the end
    (3, 512, 4, 64, 64, 1, 128, I.BF16, [512, 128, 5]),         # a fully padded sequence
    (3, 300, 4, 64, 16, 2, 64, I.F32, [0, 64, 170]),            # CUDA-core fp32 path
])
def test_left_padded_batch_matches_each_sequence_alone(b, L, H, P, N, G, Q, dt, pads):
    t = torch()
    inp = I.prefill_inputs(b, L, H, P, N, G, seed=61 + L, dtype=dt)   # padding positions hold random inputs too
    h0 = random_state((b, H, N, P), 62 + L, I.F32)
    dev = {k: to_dev(v) for k, v in inp.items()}
    pad = t.tensor(pads, dtype=t.int32, device="cuda")
    y, fs = ssd.chunk_scan_fwd(dev["x"], dev["dt_raw"], dev["dt_bias"], dev["A"], dev["B"], dev["C"], dev["D"], Q,
                               to_dev(h0), y_dtype=t.float32, pad_left=pad)
    t.cuda.synchronize()
    assert ssd.ssd_get_device_error(0)[0] == 0
    y, fs = to_host64(y), to_host64(fs)
    f = {k: I.to_f64(v) for k, v in inp.items()}
    tol = TOL_F32 if dt == I.F32 else TOL_BF16
    for i, p in enumerate(pads):
        h_init = I.to_f64(h0[i:i + 1]).copy()
        if p >= L:                                  # nothing left: the state passes through
            assert metric(fs[i:i + 1], h_init) <= tol
            continue
        sl = slice(p, L)
        y_ref, fs_ref = oracle.recurrent(f["x"][i:i + 1, sl], f["dt_raw"][i:i + 1, sl], f["dt_bias"], f["A"],
                                         f["B"][i:i + 1, sl], f["C"][i:i + 1, sl], f["D"], init_state=h_init)
        assert metric(y[i:i + 1, sl], y_ref) <= tol, (i, p)
        assert metric(fs[i:i + 1], fs_ref) <= tol, (i, p)
