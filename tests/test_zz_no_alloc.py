"""ssd_chunk_scan_fwd_noalloc: the prefill for callers that cannot allocate
device memory (its scratch is a fixed array inside the library).  Called
through the C ABI and checked against ssd_chunk_scan_fwd (caller workspace)
on the same inputs, twice in a row, within the bf16-input tolerance.  The
file name makes pytest collect it last."""
import numpy as np
import pytest

from mamba_ssd_scan_chunked_b200 import inputs as I
from mamba_ssd_scan_chunked_b200 import ssd
from tests.gpu_util import TOL_BF16, metric, to_dev, to_host64, torch

pytestmark = pytest.mark.gpu


def _ptrs(d):
    return [d[k].data_ptr() for k in ("x", "dt_raw", "dt_bias", "A", "B", "C", "D")]


def test_noalloc_matches_workspace_entry_twice():
    t = torch()
    s = I.MAMBA2_1P3B            # 4 x 2048 tokens, 64 heads, N=128: about 12.6 MiB of scratch
    inp = s.inputs()
    d = {k: to_dev(v) for k, v in inp.items()}
    desc = ssd.prefill_desc(d["x"], d["B"], s.chunk, t.float32, t.float32)
    assert ssd.ssd_chunk_scan_workspace_size(desc) <= ssd.NOALLOC_WORKSPACE_BYTES
    stream = t.cuda.current_stream().cuda_stream
    x, dt_raw, dt_bias, A, B, C, D = _ptrs(d)

    y_ref = t.empty((s.batch, s.seqlen, s.nheads, s.headdim), dtype=t.float32, device="cuda")
    f_ref = t.empty((s.batch, s.nheads, s.dstate, s.headdim), dtype=t.float32, device="cuda")
    ws = t.empty(ssd.ssd_chunk_scan_workspace_size(desc), dtype=t.uint8, device="cuda")
    assert ssd.ssd_chunk_scan_fwd(desc, x, dt_raw, dt_bias, A, B, C, D, 0, y_ref.data_ptr(), f_ref.data_ptr(),
                                  ws.data_ptr(), ws.numel(), stream) == 0
    t.cuda.synchronize()
    y_ref, f_ref = to_host64(y_ref), to_host64(f_ref)

    for call in range(2):   # the scratch keeps the previous call's contents: the second call must not care
        y = t.full((s.batch, s.seqlen, s.nheads, s.headdim), float("nan"), dtype=t.float32, device="cuda")
        f = t.full((s.batch, s.nheads, s.dstate, s.headdim), float("nan"), dtype=t.float32, device="cuda")
        st = ssd.ssd_chunk_scan_fwd_noalloc(desc, x, dt_raw, dt_bias, A, B, C, D, 0, y.data_ptr(), f.data_ptr(),
                                            stream)
        assert st == 0, ssd.STATUS.get(st, st)
        t.cuda.synchronize()
        assert ssd.ssd_get_device_error(stream)[0] == 0
        assert metric(to_host64(y), y_ref) <= TOL_BF16, call
        assert metric(to_host64(f), f_ref) <= TOL_BF16, call


def test_noalloc_rejects_problems_larger_than_its_scratch():
    t = torch()
    # 64 sequences of 8192 tokens need ~264 MiB of workspace: rejected before any launch
    desc = ssd.PrefillDesc(64, 8192, 64, 64, 128, 1, 256, ssd.SSD_BF16, ssd.SSD_F32, ssd.SSD_F32)
    assert ssd.ssd_chunk_scan_workspace_size(desc) > ssd.NOALLOC_WORKSPACE_BYTES
    dummy = t.empty(16, dtype=t.uint8, device="cuda").data_ptr()
    st = ssd.ssd_chunk_scan_fwd_noalloc(desc, dummy, dummy, 0, dummy, dummy, dummy, 0, 0, dummy + 4096, 0, 0)
    assert st == 4   # SSD_ERR_WORKSPACE
