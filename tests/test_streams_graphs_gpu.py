"""Two claims of the C ABI, on a GPU: calls on different streams with
different workspaces may run concurrently, and the calls can be captured in a
CUDA graph (the prefill's two kernels, the second a programmatic dependent of
the first, and a decode step) and replayed."""
import numpy as np
import pytest

import oracle
from mamba_ssd_scan_chunked_b200 import inputs as I
from mamba_ssd_scan_chunked_b200 import ssd
from tests.gpu_util import TOL_BF16, metric, to_dev, to_host64, torch

pytestmark = pytest.mark.gpu


def _case(seed, b=2, L=700, H=4, P=64, N=128, G=2):
    inp = I.prefill_inputs(b, L, H, P, N, G, seed=seed, dtype=I.BF16)
    f = {k: I.to_f64(v) for k, v in inp.items()}
    y_ref, fs_ref = oracle.recurrent(f["x"], f["dt_raw"], f["dt_bias"], f["A"], f["B"], f["C"], f["D"])
    return {k: to_dev(v) for k, v in inp.items()}, y_ref, fs_ref


def test_concurrent_streams_with_separate_workspaces():
    t = torch()
    cases = [_case(81), _case(82)]
    streams = [t.cuda.Stream(), t.cuda.Stream()]
    outs = []
    for (dev, _, _), s in zip(cases, streams):
        with t.cuda.stream(s):
            outs.append(ssd.chunk_scan_fwd(dev["x"], dev["dt_raw"], dev["dt_bias"], dev["A"], dev["B"], dev["C"],
                                           dev["D"], 256, y_dtype=t.float32, stream=s))
    t.cuda.synchronize()
    assert ssd.ssd_get_device_error(0)[0] == 0
    for (y, fs), (_, y_ref, fs_ref) in zip(outs, cases):
        assert metric(to_host64(y), y_ref) <= TOL_BF16
        assert metric(to_host64(fs), fs_ref) <= TOL_BF16


def test_graph_capture_and_replay():
    t = torch()
    dev, y_ref, fs_ref = _case(83)
    b, L, H, P = dev["x"].shape
    N = dev["B"].shape[3]
    y = t.empty((b, L, H, P), dtype=t.float32, device="cuda")
    fs = t.empty((b, H, N, P), dtype=t.float32, device="cuda")
    ws = t.empty(ssd.workspace_bytes(dev["x"], dev["B"], 256, t.float32, t.float32), dtype=t.uint8, device="cuda")
    step = {k: to_dev(v) for k, v in I.draw_decode_step(0, b, H, P, N, dev["B"].shape[2], seed=84,
                                                        dtype=I.BF16).items()}
    st = t.empty_like(fs)
    yd = t.empty((b, H, P), dtype=t.float32, device="cuda")
    s = t.cuda.Stream()

    def body():
        ssd.chunk_scan_fwd(dev["x"], dev["dt_raw"], dev["dt_bias"], dev["A"], dev["B"], dev["C"], dev["D"], 256,
                           y=y, final_state=fs, y_dtype=t.float32, workspace=ws, stream=s)
        st.copy_(fs)
        ssd.state_update(st, step["x"], step["dt_raw"], dev["dt_bias"], dev["A"], step["B"], step["C"], dev["D"],
                         y=yd, y_dtype=t.float32, stream=s)

    with t.cuda.stream(s):
        body()                                  # warm-up outside the capture
    s.synchronize()
    g = t.cuda.CUDAGraph()
    with t.cuda.graph(g, stream=s):
        body()
    y.zero_(); fs.zero_(); yd.zero_()
    g.replay()
    g.replay()
    t.cuda.synchronize()
    assert ssd.ssd_get_device_error(0)[0] == 0
    assert metric(to_host64(y), y_ref) <= TOL_BF16
    assert metric(to_host64(fs), fs_ref) <= TOL_BF16
    f = {k: I.to_f64(v) for k, v in I.draw_decode_step(0, b, H, P, N, dev["B"].shape[2], seed=84,
                                                        dtype=I.BF16).items()}
    hp = I.prefill_inputs(b, L, H, P, N, dev["B"].shape[2], seed=83, dtype=I.BF16)
    pf = {k: I.to_f64(v) for k, v in hp.items()}
    h = fs_ref.copy()
    yd_ref = oracle.decode_step(h, f["x"], f["dt_raw"], pf["dt_bias"], pf["A"], f["B"], f["C"], pf["D"])
    assert metric(to_host64(yd), yd_ref) <= TOL_BF16
