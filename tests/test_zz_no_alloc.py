"""ssd_chunk_scan_fwd_noalloc: the prefill for callers that cannot allocate
device memory (its scratch is a fixed array inside the library).  Called
through the C ABI and checked against ssd_chunk_scan_fwd (caller workspace) on
the same inputs, twice in a row: both run the same deterministic kernels, so
the results must be bitwise equal.  Checked against the float64 oracle
separately.  Two shapes: the head-pair kernel over whole sequences, and a few
long sequences cut into runs, whose state hand-off flags, control words and
entry-state slots live in the shared scratch; the second is also run after a
call whose hand-off waits were made to give up.  The file name makes pytest
collect it last."""
import numpy as np
import pytest

from mamba_ssd_scan_chunked_b200 import inputs as I
from mamba_ssd_scan_chunked_b200 import ssd
from tests.gpu_util import TOL_BF16, metric, oracle_prefill, to_dev, to_host64, torch

pytestmark = pytest.mark.gpu

SHAPES = {
    # 4 x 2048 tokens, 64 heads, N=128: head pairs, about 12.6 MiB of scratch
    "head_pairs_1p3b_layer": (I.MAMBA2_1P3B.inputs, 256, 2, [0, 37, 63]),
    # 2 sequences of 2048 tokens: runs of chunks handing the state on through the scratch
    "runs_with_state_handoff": (lambda: I.prefill_inputs(1, 2048, 2, 64, 128, 1, 91, I.BF16), 256, 0, None),
}


def _ptrs(d):
    return [d[k].data_ptr() for k in ("x", "dt_raw", "dt_bias", "A", "B", "C", "D")]


def _outputs(t, d, N):
    b, L, H, P = d["x"].shape
    y = t.full((b, L, H, P), float("nan"), dtype=t.float32, device="cuda")
    f = t.full((b, H, N, P), float("nan"), dtype=t.float32, device="cuda")
    return y, f


def _workspace_call(t, desc, d, N, stream):
    y, f = _outputs(t, d, N)
    ws = t.empty(ssd.ssd_chunk_scan_workspace_size(desc), dtype=t.uint8, device="cuda")
    assert ssd.ssd_chunk_scan_fwd(desc, *_ptrs(d), 0, y.data_ptr(), f.data_ptr(), ws.data_ptr(), ws.numel(),
                                  stream) == 0
    t.cuda.synchronize()
    return y, f


def _noalloc_call(t, desc, d, N, stream):
    y, f = _outputs(t, d, N)
    st = ssd.ssd_chunk_scan_fwd_noalloc(desc, *_ptrs(d), 0, y.data_ptr(), f.data_ptr(), stream)
    assert st == 0, ssd.STATUS.get(st, st)
    t.cuda.synchronize()
    return y, f


@pytest.mark.parametrize("shape", list(SHAPES))
def test_noalloc_matches_workspace_entry_twice(shape):
    t = torch()
    make, chunk, path, heads = SHAPES[shape]
    inp = make()
    d = {k: to_dev(v) for k, v in inp.items()}
    N = d["B"].shape[3]
    desc = ssd.prefill_desc(d["x"], d["B"], chunk, t.float32, t.float32)
    assert ssd.ssd_chunk_scan_path(desc) == path
    assert ssd.ssd_chunk_scan_workspace_size(desc) <= ssd.NOALLOC_WORKSPACE_BYTES
    stream = t.cuda.current_stream().cuda_stream
    y_ws, f_ws = _workspace_call(t, desc, d, N, stream)
    for call in range(2):   # the scratch keeps the previous call's contents: the second call must not care
        y, f = _noalloc_call(t, desc, d, N, stream)
        assert ssd.ssd_get_device_error(stream)[0] == 0
        assert t.equal(y, y_ws), call
        assert t.equal(f, f_ws), call
    # and the result itself against the oracle (a few heads of the large shape)
    y_ref, f_ref = oracle_prefill(inp, heads=heads)
    y64, f64 = to_host64(y_ws), to_host64(f_ws)
    if heads is not None:
        y64, f64 = y64[:, :, heads], f64[:, heads]
    assert metric(y64, y_ref) <= TOL_BF16
    assert metric(f64, f_ref) <= TOL_BF16


def test_noalloc_after_a_call_whose_handoff_waits_gave_up():
    """A call made to time out leaves the scratch's flags and abort word set; the
    next call must reset them and give the workspace entry's result exactly."""
    t = torch()
    make, chunk, path, _ = SHAPES["runs_with_state_handoff"]
    d = {k: to_dev(v) for k, v in make().items()}
    N = d["B"].shape[3]
    desc = ssd.prefill_desc(d["x"], d["B"], chunk, t.float32, t.float32)
    stream = t.cuda.current_stream().cuda_stream
    y_ws, f_ws = _workspace_call(t, desc, d, N, stream)
    assert ssd.ssd_debug_inject(ssd.SSD_FAULT_DROP_RUN_PUBLISH) == 0
    try:
        _noalloc_call(t, desc, d, N, stream)
        st, detail = ssd.ssd_get_device_error(stream)
    finally:
        assert ssd.ssd_debug_inject(0) == 0
    assert st == 6 and detail & 0x1          # SSD_ERR_DEVICE_TIMEOUT, hand-off bit
    y, f = _noalloc_call(t, desc, d, N, stream)
    assert ssd.ssd_get_device_error(stream) == (0, 0)
    assert t.equal(y, y_ws) and t.equal(f, f_ws)


def test_noalloc_rejects_problems_larger_than_its_scratch():
    t = torch()
    # 64 sequences of 8192 tokens need ~264 MiB of workspace: rejected before any launch
    desc = ssd.PrefillDesc(64, 8192, 64, 64, 128, 1, 256, ssd.SSD_BF16, ssd.SSD_F32, ssd.SSD_F32)
    assert ssd.ssd_chunk_scan_workspace_size(desc) > ssd.NOALLOC_WORKSPACE_BYTES
    dummy = t.empty(16, dtype=t.uint8, device="cuda").data_ptr()
    st = ssd.ssd_chunk_scan_fwd_noalloc(desc, dummy, dummy, 0, dummy, dummy, dummy, 0, 0, dummy + 4096, 0, 0)
    assert st == 4   # SSD_ERR_WORKSPACE
