"""GPU parity of ssd_state_update_mimo (rank-R decode) against the float64
oracle's MIMO step (itself pinned by chains of single-input steps)."""
import numpy as np
import pytest

import oracle
from mamba_ssd_scan_chunked_b200 import inputs as I
from mamba_ssd_scan_chunked_b200 import ssd
from tests.gpu_util import TOL_BF16, TOL_F32, bf16_state_metric, metric, to_dev, to_host64, torch

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("b,H,P,N,G,R", [(3, 4, 64, 128, 2, 4), (2, 6, 32, 16, 3, 2), (2, 4, 128, 64, 1, 8),
                                         (1, 2, 8, 8, 2, 1), (2, 4, 16, 256, 4, 8), (3, 5, 64, 24, 5, 2)])
@pytest.mark.parametrize("io,state", [(I.F32, I.F32), (I.BF16, I.F32), (I.BF16, I.BF16)])
def test_mimo_matches_oracle(b, H, P, N, G, R, io, state):
    t = torch()
    params = I.draw_head_params(H, seed=17)
    st0 = np.stack([I.draw_decode_state(i, H, P, N, seed=18, dtype=state) for i in range(b)])
    steps = [I.draw_mimo_step(s, b, H, P, N, G, R, seed=19, dtype=io) for s in range(4)]
    st = to_dev(st0)
    prm = {k: to_dev(v) for k, v in params.items()}
    ref = I.to_f64(st0).copy()
    f = {k: I.to_f64(v) for k, v in params.items()}
    tol = TOL_F32 if (io == I.F32 and state == I.F32) else TOL_BF16
    for s in steps:
        d = {k: to_dev(v) for k, v in s.items()}
        y = ssd.state_update_mimo(st, d["x"], d["dt_raw"], prm["dt_bias"], prm["A"], d["B"], d["C"], prm["D"],
                                  y_dtype=t.float32)
        g = {k: I.to_f64(v) for k, v in s.items()}
        y_ref = oracle.decode_step_mimo(ref, g["x"], g["dt_raw"], f["dt_bias"], f["A"], g["B"], g["C"], f["D"],
                                        round_state_bf16=(state == I.BF16))
        assert metric(to_host64(y), y_ref) <= tol
    t.cuda.synchronize()
    assert ssd.ssd_get_device_error(0)[0] == 0
    assert (bf16_state_metric if state == I.BF16 else metric)(to_host64(st), ref) <= tol


def test_rank_one_equals_state_update():
    t = torch()
    b, H, P, N, G = 2, 4, 64, 32, 2
    params = I.draw_head_params(H, seed=5)
    st0 = np.stack([I.draw_decode_state(i, H, P, N, seed=6, dtype=I.F32) for i in range(b)])
    prm = {k: to_dev(v) for k, v in params.items()}
    s1, s2 = to_dev(st0), to_dev(st0)
    for s in range(3):
        d = {k: to_dev(v) for k, v in I.draw_mimo_step(s, b, H, P, N, G, 1, seed=7, dtype=I.F32).items()}
        y1 = ssd.state_update(s1, d["x"][:, :, 0].contiguous(), d["dt_raw"], prm["dt_bias"], prm["A"],
                              d["B"][:, :, 0].contiguous(), d["C"][:, :, 0].contiguous(), prm["D"])
        y2 = ssd.state_update_mimo(s2, d["x"], d["dt_raw"], prm["dt_bias"], prm["A"], d["B"], d["C"], prm["D"])
        assert metric(to_host64(y2[:, :, 0]), to_host64(y1)) <= 1e-5
    assert metric(to_host64(s2), to_host64(s1)) <= 1e-5
