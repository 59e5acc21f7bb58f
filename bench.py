#!/usr/bin/env python
"""Benchmark of libssd (Mamba-2 SSD layer core) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one ssd_chunk_scan_fwd over the high-batch prefill workload, the
largest single-GPU configuration: batch 512 x 1024 tokens, 128 heads x P=64,
N=128, 8 groups, chunk 256; bf16 inputs, fp32 accumulation, fp32 y, and the
final state stored in bf16 for the decode hand-off.  Inputs are seeded,
synthetic and resident in HBM (x alone is 8.6 GB, far beyond the 126 MB L2).
The line's value is prefill tokens/s; the same run reports:

- "handoff_decode": the 32 ssd_state_update steps at batch 512 that the
  prefill's bf16 final state feeds (tokens/s, state GB/s);
- "decode": K decode steps at batch 256 x 128 heads with an fp32 state, with
  the same steps replayed from a checkpoint and a 16-token buffer ("replay"),
  rank-4 MIMO steps ("mimo") and Mamba-3 steps ("mamba3");
- "mamba2_1p3b": the Mamba-2 1.3B-shaped layer prefill (batch 4 x 2048 tokens,
  64 heads, 1 group), with its backward pass ("backward") and the Mamba-3
  prefill of the same layer ("mamba3");
- "workloads": the tiny fp32 prefill and the long-sequence / state-size sweep.

Timing: W untimed warm-up steps, then exactly K steps between a barrier +
cudaDeviceSynchronize on both sides, CUDA events on the launching stream, max
over ranks; SM clocks sampled with NVML during the timed region.  Multi-GPU:
one process per GPU (torchrun), each rank runs its own batch (weak scaling, no
collective on the data path); value = tokens of all ranks / max time over ranks.

--impl reference times the float64 CPU oracle (the reference arm of this
build) on a bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

# kernel paths reported by ssd_chunk_scan_path
PATH_NAMES = {0: "tensor cores", 1: "cuda cores", 2: "tensor cores, head pairs"}

METRIC = "SSD prefill tokens/s + TFLOP/s; decode tokens/s + state GB/s (1 B200)"

# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) from one
# ncu capture of each kernel, keyed by the first 16 hex digits of the SHA-256 of
# the kernel's source file at capture time and by the workload: a changed kernel
# reports null until it is captured again (summaries under profiles/).
NCU_TRAFFIC = {
    ("ssd_decode.cu", "decode_b256"): ("cba348ad46ab41a0", 1079097000 + 1024990000),
    ("ssd_prefill_pair.cu", "mamba2_1p3b"): ("b35367f961e75b78", 77953536 + 87025152),
    # captured with 32 of the 512 sequences and scaled by 16 (profiles/ssd_pair_kernel_handoff_prefill_b512.md)
    ("ssd_prefill_pair.cu", "handoff_prefill"): ("b35367f961e75b78", (729406976 + 1091555328) * 16),
}


def ncu_traffic(src: str, workload: str):
    import hashlib
    if (src, workload) not in NCU_TRAFFIC:
        return None
    path = os.path.join(ROOT, "mamba_ssd_scan_chunked_b200", "csrc", src)
    want, traffic = NCU_TRAFFIC[(src, workload)]
    try:
        with open(path, "rb") as f:
            digest = hashlib.sha256(f.read()).hexdigest()[:16]
    except OSError:
        return None
    return traffic if digest == want else None


FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ counts
def prefill_flops(b, L, H, P, N, G, Q):
    """Full-block algorithmic flops of the chunked contraction:
    b * nchunks * [G * 2 Q^2 N  (C B^T per group)  +  H * (2 Q^2 P + 4 Q N P)]."""
    nc = -(-L // Q)
    return b * nc * (G * 2 * Q * Q * N + H * (2 * Q * Q * P + 4 * Q * N * P))


def executed_flops(b, L, H, P, N, G, path, sub=128):
    """Tensor-core flops the kernels actually issue: 128-token blocks; C B^T per
    block once per pair of heads (head-pair kernel) or per head; per head C h,
    the chunk-state product and M X each twice (bf16 hi and lo parts of the
    operand computed in the kernel)."""
    nblk = -(-L // sub)
    s_per = (H // 2) if path == 2 else H
    per_head = 2 * (2 * sub * N * P) + 2 * (2 * sub * N * P) + 2 * (2 * sub * sub * P)
    return b * nblk * (s_per * 2 * sub * sub * N + H * per_head)


def prefill_bytes(b, L, H, P, N, G, io_bytes, y_bytes, state_bytes, with_init=False):
    """Algorithmic bytes: x + y + B + C + dt_raw + final_state (+ init_state)."""
    tok = b * L
    n = tok * H * P * io_bytes + tok * H * P * y_bytes + 2 * tok * G * N * io_bytes + tok * H * io_bytes
    n += b * H * N * P * state_bytes * (2 if with_init else 1)
    return n


def backward_bytes(b, L, H, P, N, G, io_bytes, grad_bytes, state_bytes):
    """Algorithmic bytes of the backward pass: x, dy, dt_raw, B, C read (io
    dtype) and dfinal_state read; dx, ddt_raw, dB, dC written (gradient dtype)."""
    tok = b * L
    ins = tok * (2 * H * P + H + 2 * G * N) * io_bytes + b * H * N * P * state_bytes
    outs = tok * (H * P + H + 2 * G * N) * grad_bytes
    return ins + outs


def backward_flops(b, L, H, P, N, G, Q):
    """Algorithmic flops of the backward, counted as the three chunked scans it
    amounts to: the state adjoint (the forward's shape) and two transposed scans
    (headdim N, dstate P, one group per head)."""
    return prefill_flops(b, L, H, P, N, G, Q) + 2 * prefill_flops(b, L, H, N, P, H, Q)


def backward_executed_flops(b, L, H, P, N, G):
    """Tensor flops the block-form backward on tensor cores executes (128-token
    blocks, hi/lo pairs): per (b, h, block) the block kernel's S^T, X dY^T (N =
    128), B Ge and C h0 (hi + lo, N = 64), Mt dY (hi + lo), dS^T C and dS B (hi +
    lo), the weighted-operand products (three per accumulator); per (b, h, block)
    and direction one rank-128 state update (hi + lo)."""
    sub = 128
    nblk = -(-L // sub)
    mm = lambda n, k: 2 * sub * n * k
    per_unit = (mm(sub, N) + mm(sub, P) + 2 * 2 * mm(P, N) + 2 * mm(P, sub) + 2 * 2 * mm(N, sub)
                + 3 * 2 * mm(N, P))
    per_state = 2 * mm(P, sub) * (N // sub)
    return b * H * nblk * (per_unit + 2 * per_state)


def decode_bytes(b, H, P, N, G, io_bytes, y_bytes, state_bytes):
    """State read + write, plus x, y, B, C, dt_raw."""
    return 2 * b * H * N * P * state_bytes + b * H * P * (io_bytes + y_bytes) + 2 * b * G * N * io_bytes + b * H * io_bytes


def roofline_of(nbytes, flops, sec, peaks, peak_kind):
    """The binding roofline (HBM bytes or bf16 tensor flops) of one call."""
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    t_tc = flops / (peaks["bf16_tflops"] * 1e12)
    gbs, tf = nbytes / sec / 1e9, flops / sec / 1e12
    if t_hbm >= t_tc:
        r = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"]}
    else:
        r = {"bound": "tensor", "achieved": tf, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
             "frac": tf / peaks["bf16_tflops"]}
    r.update({"peak_source": "measured (MEASURED_PEAKS.json)" if peak_kind == "measured" else "fallback",
              "algorithmic_bytes_per_launch": nbytes, "algorithmic_flops_per_launch": flops,
              "roofline_time_us": 1e6 * max(t_hbm, t_tc)})
    return r


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples SM clock, power and clock-event reasons with NVML every ~2 ms in a thread."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index_uuid):
        self.samples = []
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByUUID(device_index_uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # NVML unavailable: report no clocks rather than guess
            self.err = repr(e)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                pw = nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0
                self.samples.append((mhz, rs, pw))
            except Exception:
                pass
            time.sleep(0.0005)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": getattr(self, "max_mhz", None), "reasons": [],
                    "samples": 0, "note": getattr(self, "err", "no samples")}
        mhz = [s[0] for s in self.samples]
        bits = 0
        for s in self.samples:
            bits |= s[1]
        reasons = [name for bit, name in self.REASONS.items() if bits & bit and name != "gpu_idle"]
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(self.samples), "power_w_max": max(s[2] for s in self.samples)}


# ------------------------------------------------------------------ reference arm
def oracle_inputs(I, shape, batches, heads):
    """float64 oracle arguments for the listed batch elements and heads of `shape`
    (heads: whole groups, so that each keeps its own B and C)."""
    inp = shape.inputs(batches=batches)
    f = {k: I.to_f64(v) for k, v in inp.items()}
    hpg = shape.nheads // shape.ngroups
    groups = sorted({h // hpg for h in heads})
    if list(heads) != [h for g in groups for h in range(g * hpg, (g + 1) * hpg)]:
        raise ValueError("heads must be whole groups")
    return dict(x=f["x"][:, :, heads], dt_raw=f["dt_raw"][:, :, heads], dt_bias=f["dt_bias"][heads],
                A=f["A"][heads], B=f["B"][:, :, groups], C=f["C"][:, :, groups], D=f["D"][heads])


def oracle_sample_rate(oracle, args_, tok_equiv, reps_min=1, seconds=0.0):
    """float64 oracle tokens/s over prepared arguments worth `tok_equiv`
    whole-layer tokens (the (b, h) recurrences are independent).  Returns
    (tokens/s, seconds, reps)."""
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle.recurrent(**args_)
        reps += 1
        dt = time.perf_counter() - t0
        if reps >= reps_min and dt >= seconds:
            break
    return tok_equiv * reps / dt, dt, reps


def run_reference(args, rank):
    """The float64 CPU oracle on a bounded sample of the headline workload."""
    if rank != 0:
        return
    import oracle
    from mamba_ssd_scan_chunked_b200 import inputs as I
    s = I.HANDOFF_PREFILL
    heads = list(range(16))     # per step: batch element 0, the 16 heads of group 0, all 1024 tokens
    oa = oracle_inputs(I, s, [0], heads)
    tok_equiv = s.seqlen * len(heads) / s.nheads
    for _ in range(args.warmup):
        oracle.recurrent(**oa)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.recurrent(**oa)
    dt = time.perf_counter() - t0
    value = tok_equiv * args.steps / dt
    sample = (f"per step: batch element 0 of {s.batch}, heads 0-15 of {s.nheads} (group 0), all {s.seqlen} tokens "
              f"= {tok_equiv:.0f} whole-layer tokens")
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": s.name, "global_batch": s.batch, "seq_len": s.seqlen, "parallelism": "host cores"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ device inputs
def device_inputs(torch, dev, b, L, H, P, N, G, seed, io_dtype):
    """Seeded synthetic prefill inputs generated on the device with the
    workloads' value distributions: x, B, C, dt_raw ~ N(0,1); dt_bias =
    log(expm1(U[1e-3,1e-1])); A = -U[1,16]; D ~ N(0,1).  Large tensors are drawn
    in batch slices to bound the fp32 temporaries."""
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)

    def normal(shape):
        out = torch.empty(shape, dtype=io_dtype, device=dev)
        step = max(1, (1 << 28) // max(1, out[0].numel()))
        for i in range(0, shape[0], step):
            sl = out[i:i + step]
            sl.copy_(torch.randn(sl.shape, generator=gen, device=dev, dtype=torch.float32))
        return out

    u = torch.rand(H, generator=gen, device=dev) * (0.1 - 1e-3) + 1e-3
    return {"x": normal((b, L, H, P)), "dt_raw": normal((b, L, H)), "B": normal((b, L, G, N)),
            "C": normal((b, L, G, N)), "dt_bias": torch.log(torch.expm1(u)),
            "A": -(torch.rand(H, generator=gen, device=dev) * 15 + 1),
            "D": torch.randn(H, generator=gen, device=dev)}


def timed(torch, stream, call, steps, warmup, pg=None, dist=None, clocks=None):
    """ms per call of `call(k)`: warm-up calls, then exactly `steps` calls between
    events on `stream` (barrier + synchronize on both sides), max over ranks."""
    for k in range(warmup):
        call(k)
    if dist is not None:
        dist.barrier(pg)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if clocks is not None:
        clocks.__enter__()
    e0.record(stream)
    for k in range(steps):
        call(warmup + k)
    e1.record(stream)
    torch.cuda.synchronize()
    if clocks is not None:
        clocks.__exit__()
    if dist is not None:
        dist.barrier(pg)
    ms = e0.elapsed_time(e1) / steps
    return dist.max_over_ranks(pg, ms) if dist is not None else ms


# ------------------------------------------------------------------ our arm
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip timing the other benchmark workloads (tiny fp32 prefill, long-sequence sweep)")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end (host buffers) measurement")
    ap.add_argument("--workload", choices=["handoff_prefill", "mamba2_1p3b"], default="handoff_prefill",
                    help="the headline prefill workload (default: the batch-512 prefill, the largest single-GPU one)")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the headline workload's batch (a smaller case of the same shape, for profiling)")
    ap.add_argument("--only-headline", action="store_true",
                    help="time the headline prefill alone (for profiling one workload)")
    ap.add_argument("--layer-only", action="store_true",
                    help="time the 1.3B-shaped layer's legs alone: prefill, backward, Mamba-3 prefill (for profiling)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return

    import numpy as np
    import torch

    from mamba_ssd_scan_chunked_b200 import dist
    from mamba_ssd_scan_chunked_b200 import inputs as I
    from mamba_ssd_scan_chunked_b200 import ssd

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    pg = dist.init(world, rank, local_rank)
    peaks, peak_kind = load_peaks()
    stream = torch.cuda.current_stream(dev)
    uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    bf16 = torch.bfloat16

    def to_dev(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    def check(what):
        st_err, detail = ssd.ssd_get_device_error(stream.cuda_stream)
        if st_err:
            raise RuntimeError(f"device error word {detail:#x} after {what}")

    def prefill_call(d, yb, fb, wsb, desc_, strm=None):
        st = ssd.ssd_chunk_scan_fwd(desc_, d["x"].data_ptr(), d["dt_raw"].data_ptr(), d["dt_bias"].data_ptr(),
                                    d["A"].data_ptr(), d["B"].data_ptr(), d["C"].data_ptr(), d["D"].data_ptr(), 0,
                                    yb.data_ptr(), fb.data_ptr(), wsb.data_ptr(), wsb.numel(),
                                    (strm or stream).cuda_stream)
        if st:
            raise ssd.SsdError(st, "ssd_chunk_scan_fwd")


    # ================= the Mamba-2 1.3B-shaped layer: prefill, backward, Mamba-3 prefill
    def layer_legs():
        c1 = I.MAMBA2_1P3B
        my_batches = dist.shard(c1.batch * world, rank, world)
        NSETS = 3       # rotating input sets (x 67 MB each) so no step finds its inputs in L2
        sets = []
        for k in range(NSETS):
            batches = [bb + k * c1.batch * world for bb in my_batches]
            sets.append({kk: to_dev(v) for kk, v in c1.inputs(batches=batches).items()})
        y1 = torch.empty((c1.batch, c1.seqlen, c1.nheads, c1.headdim), dtype=torch.float32, device=dev)
        f1 = torch.empty((c1.batch, c1.nheads, c1.dstate, c1.headdim), dtype=torch.float32, device=dev)
        desc1 = ssd.prefill_desc(sets[0]["x"], sets[0]["B"], c1.chunk, torch.float32, torch.float32)
        path1 = ssd.ssd_chunk_scan_path(desc1)
        ws1 = torch.empty(ssd.ssd_chunk_scan_workspace_size(desc1), dtype=torch.uint8, device=dev)
        c1_steps = max(args.steps, 2000)              # about 0.2 s of calls
        c1clk = ClockSampler(uuid)
        ms1 = timed(torch, stream, lambda k: prefill_call(sets[k % NSETS], y1, f1, ws1, desc1), c1_steps,
                    args.warmup, pg, dist, c1clk)
        check("the 1.3B-layer prefill")
        t1 = c1.batch * c1.seqlen
        fl1 = prefill_flops(c1.batch, c1.seqlen, c1.nheads, c1.headdim, c1.dstate, c1.ngroups, c1.chunk)
        xf1 = executed_flops(c1.batch, c1.seqlen, c1.nheads, c1.headdim, c1.dstate, c1.ngroups, path1)
        nb1 = prefill_bytes(c1.batch, c1.seqlen, c1.nheads, c1.headdim, c1.dstate, c1.ngroups, 2, 4, 4)
        r1 = roofline_of(nb1, fl1, ms1 * 1e-3, peaks, peak_kind)
        r1.update({"traffic": ncu_traffic("ssd_prefill_pair.cu", "mamba2_1p3b"),
                   "kernel": "ssd_chunk_scan_fwd (decay cumsum + tcgen05 head-pair chunk kernel)"})
        c1_line = {"workload": c1.name, "steps": c1_steps, "tokens_per_s": t1 * world / (ms1 * 1e-3), "ms_per_step": ms1,
                   "tflops": fl1 / (ms1 * 1e-3) / 1e12, "executed_tflops": xf1 / (ms1 * 1e-3) / 1e12,
                   "executed_flops_per_call": xf1, "gbs": nb1 / (ms1 * 1e-3) / 1e9, "kernel_path": PATH_NAMES[path1],
                   "y": "fp32", "final_state": "fp32", "l2": "3 rotating input sets (x 67 MB each)",
                   "roofline": r1, "clocks": c1clk.summary()}

        # ---- backward pass of the same layer
        gen = torch.Generator(device=dev)
        gen.manual_seed(1000 + rank)
        dyb = torch.randn((c1.batch, c1.seqlen, c1.nheads, c1.headdim), generator=gen, device=dev).to(bf16)
        dfin = 0.1 * torch.randn((c1.batch, c1.nheads, c1.dstate, c1.headdim), generator=gen, device=dev)
        bws = torch.empty(ssd.ssd_chunk_scan_bwd_workspace_size(desc1), dtype=torch.uint8, device=dev)
        gx = torch.empty((c1.batch, c1.seqlen, c1.nheads, c1.headdim), dtype=torch.float32, device=dev)
        gdt = torch.empty((c1.batch, c1.seqlen, c1.nheads), dtype=torch.float32, device=dev)
        gB = torch.empty((c1.batch, c1.seqlen, c1.ngroups, c1.dstate), dtype=torch.float32, device=dev)
        gC = torch.empty_like(gB)
        gpar = torch.empty((3, c1.nheads), dtype=torch.float32, device=dev)
        launches_per_bwd = ssd.ssd_chunk_scan_bwd_launches(desc1, True)

        def backward(k):
            d = sets[k % NSETS]
            st = ssd.ssd_chunk_scan_bwd(desc1, d["x"].data_ptr(), d["dt_raw"].data_ptr(), d["dt_bias"].data_ptr(),
                                        d["A"].data_ptr(), d["B"].data_ptr(), d["C"].data_ptr(), d["D"].data_ptr(), 0,
                                        dyb.data_ptr(), dfin.data_ptr(), gx.data_ptr(), gdt.data_ptr(),
                                        gpar[0].data_ptr(), gpar[1].data_ptr(), gB.data_ptr(), gC.data_ptr(),
                                        gpar[2].data_ptr(), 0, bws.data_ptr(), bws.numel(), stream.cuda_stream)
            if st:
                raise ssd.SsdError(st, "ssd_chunk_scan_bwd")

        bsteps = max(10, min(args.steps, 50))
        bms = timed(torch, stream, backward, bsteps, args.warmup, pg, dist)
        check("the timed backward")
        bbytes = backward_bytes(c1.batch, c1.seqlen, c1.nheads, c1.headdim, c1.dstate, c1.ngroups, 2, 4, 4)
        bflops = backward_flops(c1.batch, c1.seqlen, c1.nheads, c1.headdim, c1.dstate, c1.ngroups, c1.chunk)
        broof = roofline_of(bbytes, bflops, bms * 1e-3, peaks, peak_kind)
        broof["kernel"] = ("ssd_chunk_scan_bwd (block form on tensor cores: state passes, block gradients, "
                           "dB/dC partial sums, parameter sums)")
        bexec = backward_executed_flops(c1.batch, c1.seqlen, c1.nheads, c1.headdim, c1.dstate, c1.ngroups)
        backward_line = {"tokens_per_s": t1 * world / (bms * 1e-3), "ms_per_step": bms, "steps": bsteps,
                         "launches_per_step": launches_per_bwd, "gradients": "fp32", "dfinal_state": "given",
                         "gbs": bbytes / (bms * 1e-3) / 1e9, "tflops": bflops / (bms * 1e-3) / 1e12,
                         "executed_tflops": bexec / (bms * 1e-3) / 1e12, "executed_flops_per_call": bexec,
                         "roofline": broof}
        del dyb, dfin, bws, gx, gdt, gB, gC, gpar

        # ---- Mamba-3 prefill (trapezoidal input + rotational state) of the same layer
        ex = I.draw_mamba3_extras(c1.batch, c1.seqlen, c1.nheads, c1.ngroups, c1.dstate, c1.seed + rank)
        m3_lam, m3_theta = to_dev(ex["lam"]), to_dev(ex["theta"])
        m3ws = torch.empty(ssd.ssd_chunk_scan_mamba3_workspace_size(desc1), dtype=torch.uint8, device=dev)
        launches_per_m3 = ssd.ssd_chunk_scan_mamba3_launches(desc1, True, True, True)

        def mamba3(k):
            d = sets[k % NSETS]
            st = ssd.ssd_chunk_scan_fwd_mamba3(desc1, d["x"].data_ptr(), d["dt_raw"].data_ptr(), d["dt_bias"].data_ptr(),
                                               d["A"].data_ptr(), d["B"].data_ptr(), d["C"].data_ptr(),
                                               d["D"].data_ptr(), m3_lam.data_ptr(), m3_theta.data_ptr(), 0,
                                               y1.data_ptr(), f1.data_ptr(), m3ws.data_ptr(), m3ws.numel(),
                                               stream.cuda_stream)
            if st:
                raise ssd.SsdError(st, "ssd_chunk_scan_fwd_mamba3")

        m3steps = max(10, min(args.steps, 50))
        m3ms = timed(torch, stream, mamba3, m3steps, args.warmup, pg, dist)
        check("the timed Mamba-3 prefill")
        mamba3_line = {"tokens_per_s": t1 * world / (m3ms * 1e-3), "ms_per_step": m3ms, "steps": m3steps,
                       "launches_per_step": launches_per_m3, "vs_mamba2_prefill_time": m3ms / ms1,
                       "inputs": "lam ~ U[0,1] per (token, head), theta ~ U[-0.5,0.5] rad per (token, group, pair)",
                       "path": ("B, C turned by the cumulative angle in bf16 hi/lo pairs, one head-pair scan taking "
                                "the three products and the diagonal correction"
                                if ssd.ssd_chunk_scan_path(desc1) == 2 else
                                "B, C turned by the cumulative angle in bf16 hi/lo pairs, three tensor-core scans")}
        c1_line["backward"] = backward_line
        c1_line["mamba3"] = mamba3_line
        del sets, y1, f1, ws1, m3ws
        torch.cuda.empty_cache()
        return c1_line

    if args.layer_only:
        # profiling: the 1.3B-shaped layer's legs alone (a few GB on the device)
        c1_line = layer_legs()
        if rank == 0:
            print(json.dumps({"metric": METRIC, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                              "data": "synthetic", "legs": "1.3B-shaped layer only", "mamba2_1p3b": c1_line}),
                  flush=True)
        dist.finish(pg)
        return

    # ================= headline: batch-512 prefill (each rank its own 512 sequences)
    s = I.HANDOFF_PREFILL if args.workload == "handoff_prefill" else I.MAMBA2_1P3B
    b, L, H, P, N, G, Q = s.batch, s.seqlen, s.nheads, s.headdim, s.dstate, s.ngroups, s.chunk
    if args.batch > 0:
        if not args.only_headline:
            raise SystemExit("--batch is a profiling option: use it with --only-headline")
        b = args.batch
    sdt = bf16 if s is I.HANDOFF_PREFILL else torch.float32     # the hand-off keeps the final state in bf16
    inp = device_inputs(torch, dev, b, L, H, P, N, G, 4000 + rank, bf16)
    y = torch.empty((b, L, H, P), dtype=torch.float32, device=dev)
    fs = torch.empty((b, H, N, P), dtype=sdt, device=dev)
    desc = ssd.prefill_desc(inp["x"], inp["B"], Q, torch.float32, sdt)
    path = ssd.ssd_chunk_scan_path(desc)
    ws = torch.empty(ssd.ssd_chunk_scan_workspace_size(desc), dtype=torch.uint8, device=dev)

    clk = ClockSampler(uuid)
    ms = timed(torch, stream, lambda k: prefill_call(inp, y, fs, ws, desc), args.steps, args.warmup, pg, dist, clk)
    check("the timed prefill")
    tokens_rank = b * L
    value = tokens_rank * world / (ms * 1e-3)
    flops = prefill_flops(b, L, H, P, N, G, Q)
    xflops = executed_flops(b, L, H, P, N, G, path)
    nbytes = prefill_bytes(b, L, H, P, N, G, 2, 4, 2 if sdt == bf16 else 4)
    roofline = roofline_of(nbytes, flops, ms * 1e-3, peaks, peak_kind)
    roofline.update({"traffic": ncu_traffic("ssd_prefill_pair.cu", args.workload),
                     "kernel": "ssd_chunk_scan_fwd (decay cumsum + tcgen05 head-pair chunk kernel)"})
    if args.only_headline:
        if rank == 0:
            print(json.dumps({"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
                              "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
                              "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                              "config": {"workload": s.name, "global_batch": b * world, "seq_len": L,
                                         "kernel_path": PATH_NAMES[path], "legs": "headline only"},
                              "roofline": roofline, "gpu_launches": 2 * args.steps, "clocks": clk.summary()}),
                  flush=True)
        dist.finish(pg)
        return

    # ---- the hand-off: the prefill's bf16 final state feeds 32 decode steps at batch 512
    if s is not I.HANDOFF_PREFILL:
        raise SystemExit("--workload mamba2_1p3b runs with --only-headline")
    dsh = I.HANDOFF_DECODE
    gen = torch.Generator(device=dev)
    gen.manual_seed(4100 + rank)
    nin = 8
    hsteps = [{"x": torch.randn((b, H, P), generator=gen, device=dev).to(bf16),
               "dt_raw": torch.randn((b, H), generator=gen, device=dev).to(bf16),
               "B": torch.randn((b, G, N), generator=gen, device=dev).to(bf16),
               "C": torch.randn((b, G, N), generator=gen, device=dev).to(bf16)} for _ in range(nin)]
    yd4 = torch.empty((b, H, P), dtype=torch.float32, device=dev)
    hdesc = ssd.DecodeDesc(b, H, P, N, G, ssd.SSD_BF16, ssd.SSD_F32, ssd.SSD_BF16)

    def handoff_step(k):
        d = hsteps[k % nin]
        st = ssd.ssd_state_update(hdesc, fs.data_ptr(), d["x"].data_ptr(), d["dt_raw"].data_ptr(),
                                  inp["dt_bias"].data_ptr(), inp["A"].data_ptr(), d["B"].data_ptr(),
                                  d["C"].data_ptr(), inp["D"].data_ptr(), yd4.data_ptr(), stream.cuda_stream)
        if st:
            raise ssd.SsdError(st, "ssd_state_update")

    prefill_call(inp, y, fs, ws, desc)          # a fresh final state for the hand-off
    hclk = ClockSampler(uuid)
    hms = timed(torch, stream, handoff_step, dsh.steps, 3, pg, dist, hclk)
    check("the hand-off decode")
    hbytes = decode_bytes(b, H, P, N, G, 2, 4, 2)
    hgbs = hbytes / (hms * 1e-3) / 1e9
    handoff_line = {"workload": dsh.name, "steps": dsh.steps, "tokens_per_s": b * world / (hms * 1e-3),
                    "ms_per_step": hms, "state_gbs": 2 * b * H * N * P * 2 / (hms * 1e-3) / 1e9,
                    "state": "bf16 (the prefill's final state)",
                    "roofline": {"bound": "hbm", "achieved": hgbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                 "frac": hgbs / peaks["hbm_gbs"], "traffic": None,
                                 "algorithmic_bytes_per_launch": hbytes, "kernel": "state_update_warp_kernel"},
                    "clocks": hclk.summary()}
    del hsteps, yd4

    # ---- end to end through the public API with host buffers: the batch streamed in
    # slices of 32 sequences, each slice's inputs up from pinned host memory and its
    # y and final state back, on three streams (upload of slice k+1, compute of
    # slice k, download of slice k-1 overlap; PCIe is full duplex)
    e2e = None
    if not args.no_e2e:
        SL = 32
        nsl = b // SL
        host = {k: inp[k][:SL].cpu().pin_memory() for k in ("x", "dt_raw", "B", "C")}
        y_h = torch.empty((SL, L, H, P), dtype=torch.float32).pin_memory()
        fs_h = torch.empty((SL, H, N, P), dtype=bf16).pin_memory()
        h2d_slice = sum(v.numel() * v.element_size() for v in host.values())
        d2h_slice = y_h.numel() * 4 + fs_h.numel() * 2
        sdesc = ssd.prefill_desc(inp["x"][:SL], inp["B"][:SL], Q, torch.float32, bf16)
        sws = torch.empty(ssd.ssd_chunk_scan_workspace_size(sdesc), dtype=torch.uint8, device=dev)
        s_up, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        dbuf = [{k: torch.empty_like(host[k], device=dev) for k in host} for _ in range(2)]
        for i in range(2):
            for k in ("dt_bias", "A", "D"):
                dbuf[i][k] = inp[k]
        obuf = [(torch.empty_like(y_h, device=dev), torch.empty_like(fs_h, device=dev)) for _ in range(2)]
        up_done = [torch.cuda.Event() for _ in range(2)]
        comp_done = [torch.cuda.Event() for _ in range(2)]
        down_done = [torch.cuda.Event() for _ in range(2)]
        for e_ in comp_done + down_done:
            e_.record(stream)

        def upload(k):
            i = k % 2
            s_up.wait_event(comp_done[i])           # slice k-2 has read this buffer
            with torch.cuda.stream(s_up):
                for name, v in host.items():
                    dbuf[i][name].copy_(v, non_blocking=True)
            up_done[i].record(s_up)

        def compute(k):
            i = k % 2
            stream.wait_event(up_done[i])
            stream.wait_event(down_done[i])         # slice k-2's outputs are down
            prefill_call(dbuf[i], obuf[i][0], obuf[i][1], sws, sdesc)
            comp_done[i].record(stream)

        def download(k):
            i = k % 2
            s_down.wait_event(comp_done[i])
            with torch.cuda.stream(s_down):
                y_h.copy_(obuf[i][0], non_blocking=True)
                fs_h.copy_(obuf[i][1], non_blocking=True)
            down_done[i].record(s_down)

        def run(nslices, t_start=None, t_end=None):
            if t_start is not None:
                t_start.record(s_up)
            upload(0)
            for k in range(nslices):
                if k + 1 < nslices:
                    upload(k + 1)
                compute(k)
                download(k)
            if t_end is not None:
                t_end.record(s_down)

        run(2)
        torch.cuda.synchronize()
        e2e_steps = 2                               # 2 x 16 slices: about 0.7 s of PCIe traffic
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        run(e2e_steps * nsl, ev0, ev1)
        torch.cuda.synchronize()
        check("the end-to-end prefill")
        ems = dist.max_over_ranks(pg, ev0.elapsed_time(ev1) / e2e_steps)
        e2e = {"value": tokens_rank * world / (ems * 1e-3), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d_slice * nsl, "d2h_bytes_per_step": d2h_slice * nsl, "ms_per_step": ems,
               "steps": e2e_steps,
               "pipelining": f"the batch in {nsl} slices of {SL} sequences; upload of slice k+1, compute of slice k "
                             "and download of slice k-1 overlap (3 streams)"}
        del host, y_h, fs_h, dbuf, obuf, sws

    # ---- CPU baseline: the float64 oracle on batch elements {0, 1, 255, 511}, all heads
    cpu_baseline = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        cb = [0, 1, 255, 511]
        oa = oracle_inputs(I, s, cb, list(range(H)))
        rate, cdt, reps = oracle_sample_rate(oracle, oa, len(cb) * L, reps_min=1, seconds=5.0)
        cpu_baseline = {"value": rate, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
                        "sample": f"batch elements {cb} of {b} (all {H} heads, {L} tokens each), run {reps} times "
                                  f"in {cdt:.1f} s; the (b, h) recurrences are independent, so this is the "
                                  "workload's per-token rate"}
    del inp, y, fs, ws
    torch.cuda.empty_cache()

    # ================= decode: batch 256 x 128 heads, fp32 state
    dcfg = I.DECODE_B256
    dec_batches = dist.shard(dcfg.batch * world, rank, world)
    state = torch.from_numpy(np.stack([I.draw_decode_state(bb, dcfg.nheads, dcfg.headdim, dcfg.dstate, dcfg.seed,
                                                           dcfg.state_dtype) for bb in dec_batches])).to(dev)


    prm = {k: to_dev(v) for k, v in I.draw_head_params(dcfg.nheads, dcfg.seed).items()}
    nsteps_in = 8
    dsteps = []
    for t in range(nsteps_in):
        st = I.draw_decode_step(t, dcfg.batch, dcfg.nheads, dcfg.headdim, dcfg.dstate, dcfg.ngroups, dcfg.seed,
                                dcfg.io_dtype)
        dsteps.append({k: to_dev(v) for k, v in st.items()})
    yd = torch.empty((dcfg.batch, dcfg.nheads, dcfg.headdim), dtype=torch.float32, device=dev)
    ddesc = ssd.DecodeDesc(dcfg.batch, dcfg.nheads, dcfg.headdim, dcfg.dstate, dcfg.ngroups, ssd.SSD_BF16,
                           ssd.SSD_F32, ssd.SSD_F32)

    def decode(t):
        d = dsteps[t % nsteps_in]
        st = ssd.ssd_state_update(ddesc, state.data_ptr(), d["x"].data_ptr(), d["dt_raw"].data_ptr(),
                                  prm["dt_bias"].data_ptr(), prm["A"].data_ptr(), d["B"].data_ptr(),
                                  d["C"].data_ptr(), prm["D"].data_ptr(), yd.data_ptr(), stream.cuda_stream)
        if st:
            raise ssd.SsdError(st, "ssd_state_update")

    dsteps_timed = max(dcfg.steps, args.steps)
    dclk = ClockSampler(uuid)
    dms = timed(torch, stream, decode, dsteps_timed, args.warmup, pg, dist, dclk)
    dbytes = decode_bytes(dcfg.batch, dcfg.nheads, dcfg.headdim, dcfg.dstate, dcfg.ngroups, 2, 4, 4)
    dgbs = dbytes / (dms * 1e-3) / 1e9
    decode_line = {"workload": dcfg.name, "steps": dsteps_timed, "tokens_per_s": dcfg.batch * world / (dms * 1e-3),
                   "ms_per_step": dms, "state_gbs": 2 * dcfg.batch * dcfg.nheads * dcfg.dstate * dcfg.headdim * 4
                   / (dms * 1e-3) / 1e9,
                   "roofline": {"bound": "hbm", "achieved": dgbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                "frac": dgbs / peaks["hbm_gbs"], "traffic": ncu_traffic("ssd_decode.cu", "decode_b256"),
                                "algorithmic_bytes_per_launch": dbytes, "kernel": "state_update_warp_kernel"},
                   "clocks": dclk.summary()}

    # ---- replayed decode of the same steps: checkpoint + a buffer of RK tokens, the
    # checkpoint written back once per RK steps
    RK = 16
    rdesc = ssd.ReplayDesc(dcfg.batch, dcfg.nheads, dcfg.headdim, dcfg.dstate, dcfg.ngroups, ssd.SSD_BF16,
                           ssd.SSD_F32, ssd.SSD_F32, RK)
    rbuf = torch.empty(max(ssd.ssd_replay_buffer_size(rdesc), 1), dtype=torch.uint8, device=dev)
    rfill = [0]

    def replay(t):
        d = dsteps[t % nsteps_in]
        st = ssd.ssd_replay_step(rdesc, state.data_ptr(), rbuf.data_ptr(), rfill[0], d["x"].data_ptr(),
                                 d["dt_raw"].data_ptr(), prm["dt_bias"].data_ptr(), prm["A"].data_ptr(),
                                 d["B"].data_ptr(), d["C"].data_ptr(), prm["D"].data_ptr(), yd.data_ptr(),
                                 stream.cuda_stream)
        if st:
            raise ssd.SsdError(st, "ssd_replay_step")
        rfill[0] = (rfill[0] + 1) % RK

    rsteps = RK * max(1, dsteps_timed // RK)      # whole buffer cycles: every RK-th step folds
    rms = timed(torch, stream, replay, rsteps, RK, pg, dist)
    sbytes = dcfg.batch * dcfg.nheads * dcfg.dstate * dcfg.headdim * 4
    # per step: the checkpoint read, its write once per RK steps, the step's io,
    # and the buffered x_s (per head) and B_s (per group) read back, (RK-1)/2 on average
    io_bytes = dbytes - 2 * sbytes
    buf_bytes = (RK - 1) / 2 * (dcfg.batch * dcfg.nheads * dcfg.headdim * 2
                                + dcfg.batch * dcfg.nheads * dcfg.dstate * 2)
    rbytes = sbytes * (1 + 1 / RK) + io_bytes + buf_bytes + dcfg.batch * dcfg.nheads * dcfg.headdim * 2
    rgbs = rbytes / (rms * 1e-3) / 1e9
    decode_line["replay"] = {"capacity": RK, "tokens_per_s": dcfg.batch * world / (rms * 1e-3), "ms_per_step": rms,
                             "speedup_vs_state_update": dms / rms,
                             "roofline": {"bound": "hbm", "achieved": rgbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                          "frac": rgbs / peaks["hbm_gbs"], "algorithmic_bytes_per_step": rbytes,
                                          "kernel": "replay_step_kernel"}}

    # ---- MIMO decode (rank 4) on the same state: 4x the flops of a step for the
    # same state traffic
    MR = 4
    gen = torch.Generator(device=dev)
    gen.manual_seed(dcfg.seed)
    mx_ = (torch.randn((dcfg.batch, dcfg.nheads, MR, dcfg.headdim), generator=gen, device=dev)).bfloat16()
    mB = (torch.randn((dcfg.batch, dcfg.ngroups, MR, dcfg.dstate), generator=gen, device=dev)).bfloat16()
    mC = (torch.randn((dcfg.batch, dcfg.ngroups, MR, dcfg.dstate), generator=gen, device=dev)).bfloat16()
    my_ = torch.empty((dcfg.batch, dcfg.nheads, MR, dcfg.headdim), dtype=torch.float32, device=dev)
    mdesc = ssd.MimoDesc(dcfg.batch, dcfg.nheads, dcfg.headdim, dcfg.dstate, dcfg.ngroups, MR, ssd.SSD_BF16,
                         ssd.SSD_F32, ssd.SSD_F32)

    def mimo(t):
        d = dsteps[t % nsteps_in]
        st = ssd.ssd_state_update_mimo(mdesc, state.data_ptr(), mx_.data_ptr(), d["dt_raw"].data_ptr(),
                                       prm["dt_bias"].data_ptr(), prm["A"].data_ptr(), mB.data_ptr(), mC.data_ptr(),
                                       prm["D"].data_ptr(), my_.data_ptr(), stream.cuda_stream)
        if st:
            raise ssd.SsdError(st, "ssd_state_update_mimo")

    mms = timed(torch, stream, mimo, dsteps_timed, args.warmup, pg, dist)
    check("the timed decode steps")
    mbytes = (2 * sbytes + dcfg.batch * dcfg.nheads * MR * dcfg.headdim * (2 + 4)
              + 2 * dcfg.batch * dcfg.ngroups * MR * dcfg.dstate * 2 + dcfg.batch * dcfg.nheads * 2)
    mgbs = mbytes / (mms * 1e-3) / 1e9
    decode_line["mimo"] = {"rank": MR, "tokens_per_s": dcfg.batch * world / (mms * 1e-3), "ms_per_step": mms,
                           "time_vs_state_update": mms / dms,
                           "roofline": {"bound": "hbm", "achieved": mgbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                        "frac": mgbs / peaks["hbm_gbs"], "algorithmic_bytes_per_step": mbytes,
                                        "kernel": "mimo_step_kernel"}}
    # ---- Mamba-3 decode steps on the same state: trapezoid mix lam and rotation angles
    # theta given; the previous token's x and B are the previous step's inputs
    ex3 = I.draw_mamba3_extras(dcfg.batch, nsteps_in, dcfg.nheads, dcfg.ngroups, dcfg.dstate, dcfg.seed)
    m3lam = [torch.from_numpy(np.ascontiguousarray(ex3["lam"][:, t])).to(dev) for t in range(nsteps_in)]
    m3th = [torch.from_numpy(np.ascontiguousarray(ex3["theta"][:, t])).to(dev) for t in range(nsteps_in)]

    def mamba3_step(t):
        d, dp = dsteps[t % nsteps_in], dsteps[(t - 1) % nsteps_in]
        st = ssd.ssd_state_update_mamba3(ddesc, state.data_ptr(), d["x"].data_ptr(), dp["x"].data_ptr(),
                                         d["dt_raw"].data_ptr(), prm["dt_bias"].data_ptr(), prm["A"].data_ptr(),
                                         d["B"].data_ptr(), dp["B"].data_ptr(), d["C"].data_ptr(),
                                         prm["D"].data_ptr(), m3lam[t % nsteps_in].data_ptr(),
                                         m3th[t % nsteps_in].data_ptr(), yd.data_ptr(), stream.cuda_stream)
        if st:
            raise ssd.SsdError(st, "ssd_state_update_mamba3")

    m3dms = timed(torch, stream, mamba3_step, dsteps_timed, args.warmup, pg, dist)
    check("the timed Mamba-3 decode steps")
    m3dbytes = (dbytes + dcfg.batch * dcfg.nheads * dcfg.headdim * 2 + dcfg.batch * dcfg.ngroups * dcfg.dstate * 2
                + dcfg.batch * dcfg.nheads * 4 + dcfg.batch * dcfg.ngroups * dcfg.dstate // 2 * 4)
    m3dgbs = m3dbytes / (m3dms * 1e-3) / 1e9
    decode_line["mamba3"] = {"tokens_per_s": dcfg.batch * world / (m3dms * 1e-3), "ms_per_step": m3dms,
                             "time_vs_state_update": m3dms / dms,
                             "inputs": "lam ~ U[0,1] per (b, head), theta ~ U[-0.5,0.5] rad per (b, group, pair); "
                                       "x_prev, B_prev = the previous step's x, B",
                             "roofline": {"bound": "hbm", "achieved": m3dgbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                          "frac": m3dgbs / peaks["hbm_gbs"], "algorithmic_bytes_per_step": m3dbytes,
                                          "kernel": "mamba3_step_kernel"}}
    del state, dsteps, yd, rbuf, mx_, mB, mC, my_
    torch.cuda.empty_cache()

    c1_line = layer_legs()

    # ================= the other workloads: tiny fp32 prefill, long-sequence / state-size sweep
    workloads = None
    if rank == 0 and world == 1 and not args.no_workloads:
        workloads = {}
        for sh in [I.TINY_FP32] + I.long_sequence_sweep():
            bw, Lw, Hw, Pw, Nw, Gw, Qw = sh.batch, sh.seqlen, sh.nheads, sh.headdim, sh.dstate, sh.ngroups, sh.chunk
            fp32 = sh.dtype == I.F32
            iod = torch.float32 if fp32 else bf16
            d = device_inputs(torch, dev, bw, Lw, Hw, Pw, Nw, Gw, 2, iod)
            yw = torch.empty((bw, Lw, Hw, Pw), dtype=torch.float32, device=dev)
            fw = torch.empty((bw, Hw, Nw, Pw), dtype=torch.float32, device=dev)
            dw = ssd.prefill_desc(d["x"], d["B"], Qw, torch.float32, torch.float32)
            wsw = torch.empty(max(ssd.ssd_chunk_scan_workspace_size(dw), 1), dtype=torch.uint8, device=dev)
            # about 0.2 s of calls (at least 10)
            prefill_call(d, yw, fw, wsw, dw)
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            prefill_call(d, yw, fw, wsw, dw)
            torch.cuda.synchronize()
            n = int(max(10, min(20000, 0.2 / max(time.perf_counter() - t0, 1e-6))))
            msw = timed(torch, stream, lambda k: prefill_call(d, yw, fw, wsw, dw), n, 3)
            io_b = 4 if fp32 else 2
            nbw = prefill_bytes(bw, Lw, Hw, Pw, Nw, Gw, io_b, 4, 4)
            flw = prefill_flops(bw, Lw, Hw, Pw, Nw, Gw, Qw)
            rw = roofline_of(nbw, flw, msw * 1e-3, peaks, peak_kind)
            pth = ssd.ssd_chunk_scan_path(dw)
            workloads[sh.name] = {"kind": "prefill", "path": PATH_NAMES[pth], "calls": n,
                                  "tokens_per_s": bw * Lw / (msw * 1e-3), "ms_per_call": msw,
                                  "tflops": flw / (msw * 1e-3) / 1e12, "gbs": nbw / (msw * 1e-3) / 1e9,
                                  "bound": rw["bound"], "frac": rw["frac"]}
            if fp32:
                workloads[sh.name]["note"] = "launch-bound at this size (two launches of microseconds)"
            del d, yw, fw, wsw
            torch.cuda.empty_cache()
        check("the workload sweep")

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": s.name, "global_batch": b * world, "seq_len": L, "nheads": H, "headdim": P,
                           "dstate": N, "ngroups": G, "chunk": Q, "inputs": "bf16", "accumulate": "fp32",
                           "y": "fp32", "final_state": "bf16 (fed to the decode hand-off)",
                           "parallelism": f"dp{world}" if world > 1 else "single",
                           "l2": "inputs larger than L2 (x 8.6 GB per step)", "kernel_path": PATH_NAMES[path]},
                "tflops": flops / (ms * 1e-3) / 1e12, "executed_tflops": xflops / (ms * 1e-3) / 1e12,
                "executed_flops_per_call": xflops, "gbs": nbytes / (ms * 1e-3) / 1e9, "roofline": roofline,
                "handoff_decode": handoff_line, "decode": decode_line, "mamba2_1p3b": c1_line,
                "cpu_baseline": cpu_baseline, "e2e": e2e, "workloads": workloads,
                "gpu_launches": 2 * args.steps,
                "gpu_launches_other_legs": {"handoff_decode": dsh.steps, "decode": dsteps_timed,
                                            "replay": 2 * rsteps, "mimo": dsteps_timed,
                                            "mamba3_decode": dsteps_timed, "mamba2_1p3b": 2 * c1_line["steps"],
                                            "backward": (c1_line["backward"]["launches_per_step"] *
                                                         c1_line["backward"]["steps"]),
                                            "mamba3": (c1_line["mamba3"]["launches_per_step"] *
                                                       c1_line["mamba3"]["steps"])},
                "clocks": clk.summary()}
        print(json.dumps(line), flush=True)
    dist.finish(pg)


if __name__ == "__main__":
    main()
