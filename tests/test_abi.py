"""The C ABI boundary, checked without a GPU.

libssd.so must load on a machine without a GPU, export every function
include/ssd.h declares, and reject invalid requests on the host before it
touches a device (all calls below return before any CUDA call).
"""
import ctypes
import os
import re
import subprocess

import pytest

from mamba_ssd_scan_chunked_b200 import build as B
from mamba_ssd_scan_chunked_b200 import ssd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ssd.h")

OK, INVALID, UNSUPPORTED, ALIGN, WORKSPACE = 0, 1, 2, 3, 4
FAKE = 0x7f0000000000          # 16-byte aligned fake device address (never dereferenced)


@pytest.fixture(scope="module", autouse=True)
def built():
    B.build()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ssd_[a-z0-9_]+)\s*\(", text)))


def test_header_matches_binding_exports():
    assert declared_functions() == sorted(ssd.EXPORTS)


def test_library_exports_every_declared_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", ssd.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (ssd_\w+)", out))
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(ctypes.CDLL(ssd.LIB_PATH), name)


def test_version_and_status_strings():
    assert ssd.ssd_version() == 100
    for code in range(7):
        assert ssd.ssd_status_string(code).startswith(ssd.STATUS[code])
    assert ssd.ssd_status_string(99) == "SSD_ERR_UNKNOWN"


def desc(**kw):
    d = dict(batch=2, seqlen=512, nheads=4, headdim=64, dstate=128, ngroups=2, chunk=256,
             io_dtype=ssd.SSD_BF16, y_dtype=ssd.SSD_F32, state_dtype=ssd.SSD_F32)
    d.update(kw)
    return ssd.PrefillDesc(**d)


def test_workspace_size_and_path():
    d = desc()
    n = ssd.ssd_chunk_scan_workspace_size(d)
    BH, Lpad = 2 * 4, 512
    # dt + cumsum (fp32 per token and head) + the fp32 entry state of every run after
    # the first (8 sequences of 2 chunks: 2 runs each) + flags
    assert n >= 2 * 4 * BH * Lpad + 4 * BH * 128 * 64
    assert ssd.ssd_chunk_scan_path(d) == 0                       # bf16, N=128: tensor cores
    assert ssd.ssd_chunk_scan_path(desc(io_dtype=ssd.SSD_F32)) == 1   # fp32: CUDA cores
    # pairs of heads of a group once there are >= 148 sequences and an even number of heads per group
    assert ssd.ssd_chunk_scan_path(desc(batch=2, nheads=74, ngroups=1)) == 2
    assert ssd.ssd_chunk_scan_path(desc(batch=2, nheads=74, ngroups=74)) == 0      # one head per group
    assert ssd.ssd_chunk_scan_path(desc(batch=1, nheads=146, ngroups=1)) == 0      # 146 sequences
    assert ssd.ssd_chunk_scan_path(desc(batch=4, nheads=64, ngroups=1, dstate=64)) == 0
    # the CUDA-core path keeps one fp32 state per chunk
    n32 = ssd.ssd_chunk_scan_workspace_size(desc(io_dtype=ssd.SSD_F32))
    assert n32 >= 4 * BH * 2 * 128 * 64
    # ragged sequence: chunks are rounded up
    assert ssd.ssd_chunk_scan_workspace_size(desc(seqlen=513)) > n


@pytest.mark.parametrize("kw,code", [
    (dict(nheads=4, ngroups=3), INVALID),
    (dict(batch=-1), INVALID),
    (dict(nheads=0), INVALID),
    (dict(io_dtype=7), INVALID),
    (dict(y_dtype=-1), INVALID),
    (dict(chunk=48), UNSUPPORTED),
    (dict(chunk=512), UNSUPPORTED),
    (dict(chunk=8), UNSUPPORTED),
    (dict(headdim=12), UNSUPPORTED),
    (dict(dstate=264), UNSUPPORTED),
])
def test_descriptor_validation(kw, code):
    with pytest.raises(ssd.SsdError) as e:
        ssd.ssd_chunk_scan_workspace_size(desc(**kw))
    assert e.value.status == code


def fwd(d, **ptrs):
    p = dict(x=FAKE, dt_raw=FAKE + 0x1000000, dt_bias=0, A=FAKE + 0x2000000, B=FAKE + 0x3000000,
             C=FAKE + 0x4000000, D=0, init_state=0, y=FAKE + 0x10000000, final_state=0, workspace=0,
             workspace_bytes=0, stream=0)
    p.update(ptrs)
    return ssd.ssd_chunk_scan_fwd(d, p["x"], p["dt_raw"], p["dt_bias"], p["A"], p["B"], p["C"], p["D"],
                                  p["init_state"], p["y"], p["final_state"], p["workspace"], p["workspace_bytes"],
                                  p["stream"])


def test_prefill_host_validation_codes():
    d = desc()
    assert fwd(d, x=0) == INVALID
    assert fwd(d, A=0) == INVALID
    assert fwd(d, y=0) == INVALID
    assert fwd(d, x=FAKE + 8) == ALIGN
    assert fwd(d, D=FAKE + 0x5000004) == ALIGN
    assert fwd(d, y=FAKE) == INVALID                       # y aliases x
    assert fwd(d) == WORKSPACE                             # no workspace
    need = ssd.ssd_chunk_scan_workspace_size(d)
    assert fwd(d, workspace=FAKE + 0x20000000, workspace_bytes=need - 1) == WORKSPACE
    assert fwd(d, workspace=FAKE + 0x20000010, workspace_bytes=need) == ALIGN   # workspace wants 256-byte alignment
    assert fwd(desc(batch=0)) == OK                        # empty batch: nothing to do, nothing launched
    assert fwd(desc(chunk=100)) == UNSUPPORTED


def test_decode_host_validation_codes():
    def dd(**kw):
        d = dict(batch=8, nheads=4, headdim=64, dstate=128, ngroups=2, io_dtype=ssd.SSD_BF16,
                 y_dtype=ssd.SSD_F32, state_dtype=ssd.SSD_F32)
        d.update(kw)
        return ssd.DecodeDesc(**d)

    def call(d, **ptrs):
        p = dict(state=FAKE, x=FAKE + 0x1000000, dt_raw=FAKE + 0x2000000, dt_bias=0, A=FAKE + 0x3000000,
                 B=FAKE + 0x4000000, C=FAKE + 0x5000000, D=0, y=FAKE + 0x6000000, stream=0)
        p.update(ptrs)
        return ssd.ssd_state_update(d, p["state"], p["x"], p["dt_raw"], p["dt_bias"], p["A"], p["B"], p["C"],
                                    p["D"], p["y"], p["stream"])

    assert call(dd(ngroups=3)) == INVALID
    assert call(dd(headdim=10)) == UNSUPPORTED
    assert call(dd(state_dtype=5)) == INVALID
    assert call(dd(), state=0) == INVALID
    assert call(dd(), x=FAKE + 0x1000004) == ALIGN
    assert call(dd(), y=FAKE) == INVALID                   # y overlaps the state
    assert call(dd(batch=0)) == OK


def replay_d(**kw):
    d = dict(batch=8, nheads=4, headdim=64, dstate=128, ngroups=2, io_dtype=ssd.SSD_BF16,
             y_dtype=ssd.SSD_F32, state_dtype=ssd.SSD_F32, capacity=16)
    d.update(kw)
    return ssd.ReplayDesc(**d)


def test_replay_buffer_size():
    # x [b][H][K][P] + B [b][G][K][N] (io dtype) + dt, cumsum [b][H][K] fp32 + the step's
    # C.B_s [b][G][16] fp32, each part 256-byte aligned
    b, H, P, N, G, K = 8, 4, 64, 128, 2, 16
    assert ssd.ssd_replay_buffer_size(replay_d()) == \
        b * H * K * P * 2 + b * G * K * N * 2 + 2 * b * H * K * 4 + 256 * ((b * G * 16 * 4 + 255) // 256)
    assert ssd.ssd_replay_buffer_size(replay_d(io_dtype=ssd.SSD_F32)) == \
        b * H * K * P * 4 + b * G * K * N * 4 + 2 * b * H * K * 4 + 256 * ((b * G * 16 * 4 + 255) // 256)
    assert ssd.ssd_replay_buffer_size(replay_d(batch=0)) == 0
    for kw, code in [(dict(capacity=0), INVALID), (dict(capacity=17), UNSUPPORTED), (dict(headdim=96), UNSUPPORTED),
                     (dict(headdim=256), UNSUPPORTED), (dict(dstate=12), UNSUPPORTED), (dict(ngroups=3), INVALID),
                     (dict(y_dtype=4), INVALID)]:
        with pytest.raises(ssd.SsdError) as e:
            ssd.ssd_replay_buffer_size(replay_d(**kw))
        assert e.value.status == code, kw


def test_replay_host_validation_codes():
    def call(d, fill=0, **ptrs):
        p = dict(ckpt=FAKE, buf=FAKE + 0x8000000, x=FAKE + 0x1000000, dt_raw=FAKE + 0x2000000, dt_bias=0,
                 A=FAKE + 0x3000000, B=FAKE + 0x4000000, C=FAKE + 0x5000000, D=0, y=FAKE + 0x6000000, stream=0)
        p.update(ptrs)
        return ssd.ssd_replay_step(d, p["ckpt"], p["buf"], fill, p["x"], p["dt_raw"], p["dt_bias"], p["A"], p["B"],
                                   p["C"], p["D"], p["y"], p["stream"])

    assert call(replay_d(), fill=16) == INVALID            # fill must be below the capacity
    assert call(replay_d(), fill=-1) == INVALID
    assert call(replay_d(), buf=0) == INVALID
    assert call(replay_d(), ckpt=0) == INVALID
    assert call(replay_d(), buf=FAKE + 0x8000010) == ALIGN   # the buffer wants 256-byte alignment
    assert call(replay_d(), x=FAKE + 0x1000008) == ALIGN
    assert call(replay_d(), y=FAKE) == INVALID              # y overlaps the checkpoint
    assert call(replay_d(), buf=FAKE + 0x100) == INVALID    # the buffer overlaps the checkpoint
    assert call(replay_d(headdim=48)) == UNSUPPORTED
    assert call(replay_d(batch=0)) == OK                   # nothing to do, nothing launched


def test_mimo_host_validation_codes():
    def md(**kw):
        d = dict(batch=8, nheads=4, headdim=64, dstate=128, ngroups=2, rank=4, io_dtype=ssd.SSD_BF16,
                 y_dtype=ssd.SSD_F32, state_dtype=ssd.SSD_F32)
        d.update(kw)
        return ssd.MimoDesc(**d)

    def call(d, **ptrs):
        p = dict(state=FAKE, x=FAKE + 0x1000000, dt_raw=FAKE + 0x2000000, dt_bias=0, A=FAKE + 0x3000000,
                 B=FAKE + 0x4000000, C=FAKE + 0x5000000, D=0, y=FAKE + 0x6000000, stream=0)
        p.update(ptrs)
        return ssd.ssd_state_update_mimo(d, p["state"], p["x"], p["dt_raw"], p["dt_bias"], p["A"], p["B"], p["C"],
                                         p["D"], p["y"], p["stream"])

    assert call(md(rank=3)) == UNSUPPORTED
    assert call(md(rank=16)) == UNSUPPORTED
    assert call(md(rank=0)) == INVALID
    assert call(md(headdim=256)) == UNSUPPORTED
    assert call(md(ngroups=3)) == INVALID
    assert call(md(), B=0) == INVALID
    assert call(md(), x=FAKE + 0x1000008) == ALIGN
    assert call(md(), y=FAKE + 0x1000000) == INVALID        # y overlaps x
    assert call(md(batch=0)) == OK


def test_mamba3_step_host_validation_codes():
    def dd(**kw):
        d = dict(batch=8, nheads=4, headdim=64, dstate=128, ngroups=2, io_dtype=ssd.SSD_BF16,
                 y_dtype=ssd.SSD_F32, state_dtype=ssd.SSD_F32)
        d.update(kw)
        return ssd.DecodeDesc(**d)

    def call(d, **ptrs):
        p = dict(state=FAKE, x=FAKE + 0x1000000, x_prev=FAKE + 0x1800000, dt_raw=FAKE + 0x2000000, dt_bias=0,
                 A=FAKE + 0x3000000, B=FAKE + 0x4000000, B_prev=FAKE + 0x4800000, C=FAKE + 0x5000000, D=0,
                 lam=FAKE + 0x7000000, theta=FAKE + 0x7800000, y=FAKE + 0x6000000, stream=0)
        p.update(ptrs)
        return ssd.ssd_state_update_mamba3(d, p["state"], p["x"], p["x_prev"], p["dt_raw"], p["dt_bias"], p["A"],
                                           p["B"], p["B_prev"], p["C"], p["D"], p["lam"], p["theta"], p["y"],
                                           p["stream"])

    assert call(dd(ngroups=3)) == INVALID
    assert call(dd(), x_prev=0) == INVALID                 # the previous token's x without its B
    assert call(dd(), B_prev=0) == INVALID
    assert call(dd(dstate=24, headdim=96)) == UNSUPPORTED   # 24 fp32 vectors per row do not divide 32
    assert call(dd(headdim=256)) == UNSUPPORTED            # fp32 state rows of 64 vectors
    assert call(dd(), state=0) == INVALID
    assert call(dd(), theta=FAKE + 0x7800004) == ALIGN
    assert call(dd(), y=FAKE + 0x1800000) == INVALID       # y overlaps x_prev
    assert call(dd(batch=0)) == OK
    assert call(dd(batch=0), x_prev=0, B_prev=0, lam=0, theta=0) == OK


def test_varlen_host_validation_codes():
    d = desc()
    need = ssd.ssd_chunk_scan_workspace_size(d)

    def call(pad_left, **kw):
        p = dict(x=FAKE, dt_raw=FAKE + 0x1000000, dt_bias=0, A=FAKE + 0x2000000, B=FAKE + 0x3000000,
                 C=FAKE + 0x4000000, D=0, init_state=0, y=FAKE + 0x10000000, final_state=0,
                 workspace=0, workspace_bytes=0, stream=0)
        p.update(kw)
        return ssd.ssd_chunk_scan_fwd_varlen(d, p["x"], p["dt_raw"], p["dt_bias"], p["A"], p["B"], p["C"], p["D"],
                                             p["init_state"], pad_left, p["y"], p["final_state"], p["workspace"],
                                             p["workspace_bytes"], p["stream"])

    assert call(0) == INVALID                              # pad_left is required
    assert call(FAKE + 0x30000002) == ALIGN                # int32 array: 4-byte aligned
    assert call(FAKE + 0x30000000) == WORKSPACE            # otherwise the checks of ssd_chunk_scan_fwd
    assert need > 0


def bwd(d, **ptrs):
    # distinct 16 MB windows per tensor (the test shapes stay far below that)
    names = ("x", "dt_raw", "dt_bias", "A", "B", "C", "D", "init_state", "dy", "dfinal_state", "dx", "ddt_raw",
             "ddt_bias", "dA", "dB", "dC", "dD", "dinit_state")
    p = {k: FAKE + 0x1000000 * i for i, k in enumerate(names)}
    for k in ("dt_bias", "D", "init_state", "dfinal_state", "ddt_bias", "dD", "dinit_state"):
        p[k] = 0
    p.update(workspace=0, workspace_bytes=0, stream=0)
    p.update(ptrs)
    return ssd.ssd_chunk_scan_bwd(d, *(p[k] for k in names), p["workspace"], p["workspace_bytes"], p["stream"])


def test_backward_workspace_and_launches():
    d = desc()
    n = ssd.ssd_chunk_scan_bwd_workspace_size(d)
    b, L, H, P, N = 2, 512, 4, 64, 128
    # bf16, dstate 128, headdim 64, an even number of heads per group: the block
    # form on tensor cores (state passes, block gradients, dB / dC partial sums,
    # parameter sums); its workspace holds bf16 hi/lo entry states and end
    # adjoints of every 128-token block
    assert ssd.ssd_chunk_scan_bwd_launches(d, False) == 4
    assert ssd.ssd_chunk_scan_bwd_launches(d, True) == 4
    assert n >= 2 * 2 * 2 * b * H * (L // 128) * N * P
    # other bf16 shapes: three chunked scans on tensor cores (dstate 256 in four
    # 64-column slices for the transposed scans)
    d256 = desc(dstate=256)
    assert ssd.ssd_chunk_scan_bwd_launches(d256, False) == 1 + 4 * 2 + 2 + 4 * 2 + 3
    n256 = ssd.ssd_chunk_scan_bwd_workspace_size(d256)
    assert n256 >= 4 * b * L * H * P + 2 * 4 * b * L * H * 256
    # fp32 inputs: the block form on CUDA cores (state passes, blocks, parameter sums)
    assert ssd.ssd_chunk_scan_bwd_launches(desc(io_dtype=ssd.SSD_F32), False) == 3
    # its workspace: fp32 entry states and end adjoints of every 32-token block
    nb = -(-L // 32)
    assert ssd.ssd_chunk_scan_bwd_workspace_size(desc(io_dtype=ssd.SSD_F32)) >= 2 * 4 * b * H * nb * N * P
    with pytest.raises(ssd.SsdError) as e:
        ssd.ssd_chunk_scan_bwd_workspace_size(desc(chunk=100))
    assert e.value.status == UNSUPPORTED


def test_backward_host_validation_codes():
    d = desc()
    need = ssd.ssd_chunk_scan_bwd_workspace_size(d)
    ws = FAKE + 0x40000000
    assert bwd(d, x=0) == INVALID
    assert bwd(d, dy=0) == INVALID
    assert bwd(d, dA=0) == INVALID
    assert bwd(d, dB=0) == INVALID
    assert bwd(d, dy=FAKE + 0x8000008) == ALIGN
    assert bwd(d, dx=FAKE) == INVALID                            # dx aliases x
    assert bwd(d, dC=FAKE + 0xa000000) == INVALID                # dC aliases dx
    assert bwd(d, dD=FAKE + 0xd000000) == INVALID                # dD aliases dA
    assert bwd(d) == WORKSPACE
    assert bwd(d, workspace=ws, workspace_bytes=need - 1) == WORKSPACE
    assert bwd(d, workspace=ws + 16, workspace_bytes=need) == ALIGN
    assert bwd(desc(chunk=100)) == UNSUPPORTED
    assert bwd(desc(nheads=4, ngroups=3)) == INVALID


def test_mamba3_workspace_launches_and_validation():
    d = desc()
    n = ssd.ssd_chunk_scan_mamba3_workspace_size(d)
    assert n > ssd.ssd_chunk_scan_workspace_size(d)
    # bf16, tensor-core path: angle sums + rotation, weights, three scans of the
    # hi/lo operands (two after a flag clear), combination, final-state rotation
    assert ssd.ssd_chunk_scan_mamba3_launches(d, True, True, True) == 2 + 1 + 1 + 2 * 2 + 1 + 1
    assert ssd.ssd_chunk_scan_mamba3_launches(d, True, False, True) == 3
    assert ssd.ssd_chunk_scan_mamba3_launches(d, False, True, False) == 2 + 1 + 1 + 2 * 2 + 1
    assert ssd.ssd_chunk_scan_mamba3_launches(d, False, False, True) == 2       # the plain forward
    assert ssd.ssd_chunk_scan_mamba3_launches(desc(io_dtype=ssd.SSD_F32), True, True, True) == 8
    # 148 or more heads in all: the head-pair kernel's Mamba-3 form takes the three
    # products and the trapezoid's own-token weights in one scan, and turns the
    # final state back as it stores it (angle sums, rotation, weights, the scan)
    dp = desc(nheads=80, ngroups=4)
    assert ssd.ssd_chunk_scan_path(dp) == 2
    assert ssd.ssd_chunk_scan_mamba3_launches(dp, True, True, True) == 4
    assert ssd.ssd_chunk_scan_mamba3_launches(dp, False, True, False) == 4
    assert ssd.ssd_chunk_scan_mamba3_launches(dp, True, False, True) == 3

    def call(dd, **kw):
        p = dict(x=FAKE, dt_raw=FAKE + 0x1000000, dt_bias=0, A=FAKE + 0x2000000, B=FAKE + 0x3000000,
                 C=FAKE + 0x4000000, D=0, lam=FAKE + 0x5000000, theta=FAKE + 0x6000000, init_state=0,
                 y=FAKE + 0x10000000, final_state=0, workspace=0, workspace_bytes=0, stream=0)
        p.update(kw)
        return ssd.ssd_chunk_scan_fwd_mamba3(dd, p["x"], p["dt_raw"], p["dt_bias"], p["A"], p["B"], p["C"], p["D"],
                                             p["lam"], p["theta"], p["init_state"], p["y"], p["final_state"],
                                             p["workspace"], p["workspace_bytes"], p["stream"])

    assert call(d) == WORKSPACE
    assert call(d, lam=FAKE + 0x5000004) == ALIGN
    assert call(d, theta=FAKE + 0x6000008) == ALIGN
    assert call(d, y=FAKE + 0x5000000) == INVALID                # y overlaps lam
    assert call(d, x=0) == INVALID
    assert call(d, y=FAKE) == INVALID                            # y aliases x
    assert call(d, workspace=FAKE + 0x40000000, workspace_bytes=n - 1) == WORKSPACE
    assert call(d, workspace=FAKE + 0x40000010, workspace_bytes=n) == ALIGN
    assert call(desc(chunk=100)) == UNSUPPORTED
    assert call(desc(batch=0)) == OK                             # nothing to do, nothing launched


def test_binding_rejects_host_or_strided_tensors_before_any_cuda_call():
    """The wrappers check devices, contiguity and the fp32 extras on the host."""
    import torch
    x = torch.zeros(1, 4, 2, 8, dtype=torch.bfloat16)
    dt = torch.zeros(1, 4, 2, dtype=torch.bfloat16)
    B = torch.zeros(1, 4, 1, 8, dtype=torch.bfloat16)
    A = torch.zeros(2)
    for call in (lambda: ssd.chunk_scan_fwd(x, dt, None, A, B, B, None, 16),
                 lambda: ssd.chunk_scan_bwd(x, dt, None, A, B, B, None, 16, x),
                 lambda: ssd.chunk_scan_fwd_mamba3(x, dt, None, A, B, B, None, 16),
                 lambda: ssd.chunk_scan_fwd_mamba3(x, dt, None, A, B, B, None, 16,
                                                   lam=torch.zeros(1, 4, 2).transpose(1, 2))):
        with pytest.raises(ValueError):
            call()


def test_binding_rejects_outputs_and_inputs_the_descriptor_does_not_describe():
    """The C ABI sizes every buffer from the descriptor; the wrappers refuse a
    tensor of another shape or dtype (a bf16 final state given where the
    descriptor says fp32 would be written past its end), before any CUDA call,
    and take y's and the final state's dtypes from the tensors given."""
    import torch
    b, L, H, P, N, G = 1, 4, 2, 8, 8, 1
    x = torch.zeros(b, L, H, P, dtype=torch.bfloat16)
    dt = torch.zeros(b, L, H, dtype=torch.bfloat16)
    B = torch.zeros(b, L, G, N, dtype=torch.bfloat16)
    A = torch.zeros(H)
    bad = [
        dict(final_state=torch.zeros(b, H, N, P, dtype=torch.bfloat16), state_dtype=torch.float32),
        dict(y=torch.zeros(b, L, H, P, dtype=torch.float32), y_dtype=torch.bfloat16),
        dict(y=torch.zeros(b, L, H, P + 1)),
        dict(final_state=torch.zeros(b, H, N + 1, P)),
    ]
    for kw in bad:
        with pytest.raises(ValueError, match="y|final_state"):
            ssd.chunk_scan_fwd(x, dt, None, A, B, B, None, 16, **kw)
    with pytest.raises(ValueError, match="dt_raw"):
        ssd.chunk_scan_fwd(x, dt.float(), None, A, B, B, None, 16)
    with pytest.raises(ValueError, match="C"):
        ssd.chunk_scan_fwd(x, dt, None, A, B, B[:, :, :, :4].contiguous(), None, 16)
    with pytest.raises(ValueError, match="A"):
        ssd.chunk_scan_fwd(x, dt, None, torch.zeros(H + 1), B, B, None, 16)
    with pytest.raises(ValueError, match="dy"):
        ssd.chunk_scan_bwd(x, dt, None, A, B, B, None, 16, x[:, :2].contiguous())
    with pytest.raises(ValueError, match="theta"):
        ssd.chunk_scan_fwd_mamba3(x, dt, None, A, B, B, None, 16, theta=torch.zeros(b, L, G, N))
    # decode: state, y and the step's operands
    st = torch.zeros(b, H, N, P)
    xd, dtd, Bd = torch.zeros(b, H, P, dtype=torch.bfloat16), torch.zeros(b, H, dtype=torch.bfloat16), \
        torch.zeros(b, G, N, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="state"):
        ssd.state_update(torch.zeros(b, H, N, P + 1), xd, dtd, None, A, Bd, Bd, None)
    with pytest.raises(ValueError, match="y"):
        ssd.state_update(st, xd, dtd, None, A, Bd, Bd, None, y=torch.zeros(b, H, P), y_dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="B_prev"):
        ssd.state_update_mamba3(st, xd, dtd, None, A, Bd, Bd, None, B_prev=torch.zeros(b, G, N + 2,
                                                                                        dtype=torch.bfloat16))
    # well-formed host tensors still reach the device check
    with pytest.raises(ValueError, match="CUDA"):
        ssd.chunk_scan_fwd(x, dt, None, A, B, B, None, 16, final_state=torch.zeros(b, H, N, P, dtype=torch.bfloat16))
