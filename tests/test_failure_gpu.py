"""Device-side failure path of the tensor-core prefill, exercised without a GPU
fault.

The prefill hands the fp32 state from one run of chunks to the next run of the
same sequence through a flag and a bounded wait (2 s).  With the test hook
SSD_FAULT_DROP_RUN_PUBLISH no run signals its successor, so the successors'
waits expire: the launch must still complete, report SSD_ERR_DEVICE_TIMEOUT with
the hand-off bit through ssd_get_device_error, and leave the context usable --
the next launch without the fault matches the oracle and reports no error.
"""
import time

import numpy as np
import pytest

from mamba_ssd_scan_chunked_b200 import inputs as I
from mamba_ssd_scan_chunked_b200 import ssd
from tests.gpu_util import TOL_BF16, gpu_prefill, metric, oracle_prefill, to_dev, torch

pytestmark = pytest.mark.gpu

ERR_CHAIN_TIMEOUT = 0x1


def test_dropped_state_handoff_times_out_and_recovers():
    # few (b, h) sequences: each is cut into runs chained through the state hand-off
    b, L, H, P, N, G, Q = 1, 2048, 2, 64, 128, 1, 256
    inp = I.prefill_inputs(b, L, H, P, N, G, 91, I.BF16)
    st, _ = ssd.ssd_get_device_error(0)
    assert st == 0
    dev = {k: to_dev(v) for k, v in inp.items()}
    desc = ssd.prefill_desc(dev["x"], dev["B"], Q)
    assert ssd.ssd_chunk_scan_path(desc) == 0
    assert ssd.ssd_debug_inject(ssd.SSD_FAULT_DROP_RUN_PUBLISH) == 0
    try:
        t0 = time.time()
        ssd.chunk_scan_fwd(dev["x"], dev["dt_raw"], dev["dt_bias"], dev["A"], dev["B"], dev["C"], dev["D"], Q)
        st, detail = ssd.ssd_get_device_error(0)     # synchronises the stream
        elapsed = time.time() - t0
    finally:
        assert ssd.ssd_debug_inject(0) == 0
    assert st == 6                                   # SSD_ERR_DEVICE_TIMEOUT
    assert detail & ERR_CHAIN_TIMEOUT
    assert elapsed < 30.0                            # a bounded wait, not a hang
    torch().cuda.synchronize()                       # the context is still usable
    # the error word was read and cleared; run again without the fault
    y, fs = gpu_prefill(inp, Q)
    y_ref, fs_ref = oracle_prefill(inp)
    assert metric(y, y_ref) <= TOL_BF16
    assert metric(fs, fs_ref) <= TOL_BF16
    st, detail = ssd.ssd_get_device_error(0)
    assert st == 0 and detail == 0


def test_debug_inject_rejects_unknown_bits():
    assert ssd.ssd_debug_inject(0x80) == 1   # SSD_ERR_INVALID_ARG
    assert ssd.ssd_debug_inject(0) == 0
