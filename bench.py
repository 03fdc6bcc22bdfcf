#!/usr/bin/env python
"""Benchmark of the chunkwise Gated DeltaNet hot path on B200.

One step = one Gated DeltaNet bf16 prefill over the 8 x 16 x 4096 x 128 batch
(chunk 64, zero initial state, fp32 output and final state) through the C ABI, with
inputs resident in HBM. Prints ONE JSON line on rank 0 with the headline tokens/s,
the roofline of that kernel, the end-to-end number through host buffers, the other
rows of the path (plain linear attention prefill, long-context prefill, the decode
step) with their own rooflines, and the fp64 oracle timed on the host cores.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1: launched with torchrun, one process per GPU; every rank runs its own batch
(weak scaling, no collective on the data path); the time is the max over ranks.
``--impl reference`` times the fp64 CPU oracle on the same workload instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gated_deltanet_sequence_b200 import workloads as W  # noqa: E402

METRIC = "chunkwise GDN prefill tokens/s + % bf16 tensor peak; decode state GB/s vs HBM"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------------- helpers
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


FP32_CLOCK_GHZ = 1.965   # B200 max SM clock (clocks.max.sm 1965 MHz)


def flops_per_head_token(mode: str, dk: int, dv: int, C: int) -> float:
    """Algorithmic FLOPs per head-token of the chunk form (dense tiles, T solve excluded):
    GDN  2C(3dk + 2dv) + 6 dk dv  (Gram [K;Q]K^T, W, U, [W;Q]S, P Ut, K~^T Ut)
    LA   2C(dk + dv) + 4 dk dv    (Q K^T, P V, Q S, K~^T V)"""
    if mode == "gdn":
        return 2 * C * (3 * dk + 2 * dv) + 6 * dk * dv
    return 2 * C * (dk + dv) + 4 * dk * dv


def prefill_bytes(B, H, L, dk, dv, in_bytes, delta, gated, s0, s_final, out_bytes=4) -> float:
    """Algorithmic HBM bytes of one prefill launch: each input read once, each output written once
    (o in fp32, out_bytes = 4, or bf16, out_bytes = 2)."""
    n = B * H * L
    b = n * (2 * dk + dv) * in_bytes + n * dv * out_bytes
    b += n * 4 * (int(delta) + int(gated))
    b += B * H * dk * dv * 4 * (int(s0) + int(s_final))
    return float(b)


def decode_bytes(N, H, dk, dv, in_bytes, delta=True, gated=True) -> float:
    """Per decode step: state read + write, q, k, v read, o written, beta / g read."""
    nh = N * H
    return float(nh * (2 * dk * dv * 4 + (2 * dk + dv) * in_bytes + dv * 4 + 4 * (int(delta) + int(gated))))


class ClockSampler:
    """Polls SM clock and throttle reasons through NVML while the timed region runs."""
    HW = 0x8  # hw_slowdown
    HW_THERMAL = 0x40
    SW_THERMAL = 0x20
    SW_POWER = 0x4

    def __init__(self, index: int, period_s: float = 0.001):
        self.samples, self.reasons, self.max_mhz = [], 0, None
        self._stop = threading.Event()
        self._period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
                self.reasons |= self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            except Exception:
                pass
            time.sleep(self._period)

    def __enter__(self):
        if self._nv is not None:
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._nv is not None:
            self._t.join()

    def summary(self):
        names = []
        for bit, name in ((self.HW, "hw_slowdown"), (self.HW_THERMAL, "hw_thermal_slowdown"),
                          (self.SW_THERMAL, "sw_thermal_slowdown"), (self.SW_POWER, "sw_power_cap")):
            if self.reasons & bit:
                names.append(name)
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


def timed(fn, steps: int, warmup: int, barrier=None):
    """ms per step of ``fn`` over exactly ``steps`` calls, CUDA events on the current stream."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    if barrier:
        barrier()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    e1.synchronize()
    torch.cuda.synchronize()
    if barrier:
        barrier()
    return e0.elapsed_time(e1) / steps


def kernel_source_hash(cu_name: str) -> str:
    """sha256[:16] of a kernel's .cu file followed by every shared header of csrc/ (sorted), so
    a change to the kernel or to any device code it may include changes the hash."""
    csrc = os.path.join(ROOT, "gated_deltanet_sequence_b200", "csrc")
    h = hashlib.sha256()
    for name in [cu_name] + sorted(f for f in os.listdir(csrc) if f.endswith(".cuh")):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_from_profiles(kernel_key: str):
    """DRAM bytes per launch recorded by an ncu capture (profiles/ncu_traffic.txt) when the
    kernel source is unchanged since the capture (kernel_source_hash); else None."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        for line in f:
            tok = line.split("#")[0].split()
            if len(tok) >= 4 and tok[0] == kernel_key:
                src = os.path.join(ROOT, "gated_deltanet_sequence_b200", "csrc", tok[1])
                if not os.path.exists(src):
                    return None
                return float(tok[3]) if kernel_source_hash(tok[1]) == tok[2] else None
    return None


# ------------------------------------------------------------------------- our arm
# ------------------------------------------------------------------------- ranks
def rank_seed(rank: int) -> int:
    """Seed of this rank's own batch of the headline workload: ranks process independent
    batches (weak scaling), so no data-path collective is needed."""
    return W.SEED_BASE + 2 + 1000 * rank


def rank_collectives(world: int, device=None):
    """(barrier, max_over_ranks) over the default process group; (None, identity) for one
    rank. ``device`` holds the reduction tensor: the GPU for NCCL, None (CPU) for gloo."""
    if world <= 1:
        return None, (lambda x: x)
    import torch.distributed as dist

    def barrier():
        dist.barrier()

    def max_over_ranks(x):
        t = torch.tensor([float(x)], device=device if device is not None else "cpu")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())
    return barrier, max_over_ranks


def aggregate_tokens_per_s(tokens_per_rank: int, world: int, ms_max: float) -> float:
    """Whole-job throughput: every rank's tokens over the slowest rank's time."""
    return world * tokens_per_rank / (ms_max * 1e-3)


def headline_config(world: int) -> dict:
    """The ``config`` of the JSON line: the headline workload, identical in both arms."""
    w = W.WORKLOADS[2]
    return {"workload": w.name, "B": w.B, "H": w.H, "L": w.L, "dk": w.dk, "dv": w.dv, "chunk": w.chunk,
            "global_batch": w.B * world, "seq_len": w.L, "parallelism": f"independent batches x{world}",
            "l2": "inputs (403 MB) and outputs (277 MB) exceed the 126 MB L2"}


def run_ours(args, rank, world, barrier, max_over_ranks):
    from gated_deltanet_sequence_b200 import _lib as gdn
    peaks, peak_src = load_peaks()
    w = W.WORKLOADS[2]
    B, H, L, dk, dv, C = w.B, w.H, w.L, w.dk, w.dv, w.chunk
    inp = W.make_prefill_inputs(B, H, L, dk, dv, mode="gdn", in_dtype=torch.bfloat16,
                                seed=rank_seed(rank), device="cuda")
    q, k, v, beta, g = inp["q"], inp["k"], inp["v"], inp["beta"], inp["g"]
    o = torch.empty(B, H, L, dv, device="cuda")
    sf = torch.empty(B, H, dk, dv, device="cuda")

    def step():
        gdn.gdn_chunk_fwd(q, k, v, beta, g, o=o, s0=None, s_final=sf, chunk=C)

    dev_index = torch.cuda.current_device()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if gdn.gdn_sync_status() != 0:
        raise RuntimeError("prefill kernel reported a device-side timeout")
    with ClockSampler(dev_index) as clk:
        ms = timed(step, args.steps, 0, barrier)
    ms_max = max_over_ranks(ms)
    # the same launch over a longer timed region (steadier clocks), reported beside the value
    long_steps = 0 if args.quick else 200
    stability = None
    if long_steps:
        with ClockSampler(dev_index) as clk_long:
            ms_long = max_over_ranks(timed(step, long_steps, 0, barrier))
        stability = {"launches": long_steps, "ms_per_launch": round(ms_long, 5), "clocks": clk_long.summary()}
    tokens = B * L
    value = aggregate_tokens_per_s(tokens, world, ms_max)
    flop = flops_per_head_token("gdn", dk, dv, C) * B * H * L
    nbytes = prefill_bytes(B, H, L, dk, dv, 2, True, True, False, True)
    gbs = nbytes / (ms * 1e-3) / 1e9
    tfs = flop / (ms * 1e-3) / 1e12
    roofline = {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(gbs / peaks["hbm_gbs"], 4),
                "traffic": traffic_from_profiles("gdn_prefill_tc"), "peak_source": peak_src,
                "kernel": "gdn prefill", "algorithmic_bytes_per_launch": nbytes}
    tensor = {"achieved": round(tfs, 1), "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
              "frac": round(tfs / peaks["bf16_tflops"], 4), "peak_source": peak_src,
              "algorithmic_flop_per_launch": flop}

    # ---- end to end through host buffers: H2D inputs, kernel, D2H outputs, every step
    e2e = None
    if not args.no_e2e:
        hq, hk, hv = (x.cpu().pin_memory() for x in (q, k, v))
        hb, hg = beta.cpu().pin_memory(), g.cpu().pin_memory()
        ho = torch.empty(B, H, L, dv, pin_memory=True)
        hs = torch.empty(B, H, dk, dv, pin_memory=True)
        dq, dk_, dv_ = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        db, dg = torch.empty_like(beta), torch.empty_like(g)

        from gated_deltanet_sequence_b200.host import gdn_chunk_fwd_host
        staging = torch.empty(int(gdn.lib.gdn_chunk_fwd_host_staging_bytes(B, H, L, dk, dv, 1, gdn.GDN_BF16, 1, 0, 1)),
                              dtype=torch.uint8, device="cuda")

        def e2e_step():
            # host buffers in, host buffers out through the C ABI call gdn_chunk_fwd_host: one
            # sequence per stage, copies overlapped with compute on the library's streams
            gdn_chunk_fwd_host(hq, hk, hv, hb, hg, o=ho, s_final=hs, chunk=C, group=1, staging=staging)

        def e2e_serial_step():
            # the same with the copies and the call in series on one stream (for comparison)
            for d, h in ((dq, hq), (dk_, hk), (dv_, hv), (db, hb), (dg, hg)):
                d.copy_(h, non_blocking=True)
            gdn.gdn_chunk_fwd(dq, dk_, dv_, db, dg, o=o, s0=None, s_final=sf, chunk=C)
            ho.copy_(o, non_blocking=True)
            hs.copy_(sf, non_blocking=True)

        e_steps = max(3, min(args.steps, 10))
        ms_e = max_over_ranks(timed(e2e_step, e_steps, 2, barrier))
        ms_serial = max_over_ranks(timed(e2e_serial_step, e_steps, 2, barrier))
        h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv, hb, hg))
        d2h = ho.numel() * 4 + hs.numel() * 4
        e2e = {"value": round(aggregate_tokens_per_s(tokens, world, ms_e), 1), "unit": "tokens/s",
               "ms_per_step": round(ms_e, 4), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "api": "gdn_chunk_fwd_host (C ABI; pinned host buffers, copies overlapped with compute)",
               "serial_ms_per_step": round(ms_serial, 4)}
        del hq, hk, hv, hb, hg, ho, hs, dq, dk_, dv_, db, dg, staging

    rows = {}
    if rank == 0 and not args.no_rows:
        del inp, q, k, v, beta, g, o, sf
        torch.cuda.empty_cache()
        rows = measure_rows(gdn, peaks, peak_src, args)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline(args.cpu_seconds)

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_max, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; q,k unit-norm, v~N(0,1), beta=sigmoid(N(0,1)), log-alpha~U(-0.05,0))",
        "config": headline_config(world),
        "roofline": roofline, "tensor": tensor, "clocks": clk.summary(), "long_region": stability,
        "e2e": e2e, "gpu_launches": args.steps, "head_tokens_per_s": round(value * H, 1),
        "rows": rows, "cpu_baseline": cpu,
    }
    return line


def measure_rows(gdn, peaks, peak_src, args):
    rows = {}
    # plain linear attention, 4 x 16 x 4096 x 128
    w = W.WORKLOADS[1]
    inp = W.make_workload_inputs(w, device="cuda")
    o = torch.empty(w.B, w.H, w.L, w.dv, device="cuda")
    fn = lambda: gdn.lin_attn_chunk_fwd(inp["q"], inp["k"], inp["v"], None, o=o, chunk=w.chunk)
    ms = timed(fn, max(5, args.steps), 3)
    nb = prefill_bytes(w.B, w.H, w.L, w.dk, w.dv, 2, False, False, False, False)
    fl = flops_per_head_token("la", w.dk, w.dv, w.chunk) * w.B * w.H * w.L
    rows["la_prefill"] = _row(w, ms, nb, fl, peaks, peak_src, "hbm", w.B * w.L, "lin_attn_tc")
    # the same with the bf16 output option (half the output bytes)
    ob = torch.empty(w.B, w.H, w.L, w.dv, device="cuda", dtype=torch.bfloat16)
    fn = lambda: gdn.lin_attn_chunk_fwd(inp["q"], inp["k"], inp["v"], None, o=ob, chunk=w.chunk)
    ms = timed(fn, max(5, args.steps), 3)
    nb = prefill_bytes(w.B, w.H, w.L, w.dk, w.dv, 2, False, False, False, False, out_bytes=2)
    rows["la_prefill_bf16_out"] = _row(w, ms, nb, fl, peaks, peak_src, "hbm", w.B * w.L)
    del inp, o, ob
    # Gated DeltaNet 8 x 16 x 4096 x 128 with both output options: bf16 o and the skip term
    w = W.WORKLOADS[2]
    inp = W.make_workload_inputs(w, device="cuda")
    D = W.make_dskip(w.H, w.dv, seed=W.SEED_BASE + 6, device="cuda")
    ob = torch.empty(w.B, w.H, w.L, w.dv, device="cuda", dtype=torch.bfloat16)
    sf = torch.empty(w.B, w.H, w.dk, w.dv, device="cuda")
    fn = lambda: gdn.gdn_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["g"], o=ob, s_final=sf,
                                   chunk=w.chunk, d_skip=D)
    ms = timed(fn, max(5, args.steps), 3)
    nb = prefill_bytes(w.B, w.H, w.L, w.dk, w.dv, 2, True, True, False, True, out_bytes=2) + w.H * w.dv * 4
    fl = flops_per_head_token("gdn", w.dk, w.dv, w.chunk) * w.B * w.H * w.L
    rows["gdn_prefill_bf16_out_skip"] = _row(w, ms, nb, fl, peaks, peak_src, "hbm", w.B * w.L)
    del ob
    # the same workload with vector-valued gates (one log-decay per token and key coordinate): a
    # per-chunk prep kernel on every SM and a per-head chain kernel, through a chunk-record
    # workspace (the call's algorithmic bytes count g in fp32 per key coordinate)
    gv = W.make_gate_per_key((w.B, w.H), w.L, w.dk, seed=W.SEED_BASE + 7, device="cuda")
    o = torch.empty(w.B, w.H, w.L, w.dv, device="cuda")
    fn = lambda: gdn.gdn_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["beta"], gv, o=o, s_final=sf, chunk=w.chunk)
    ms = timed(fn, max(5, args.steps), 3)
    nb = prefill_bytes(w.B, w.H, w.L, w.dk, w.dv, 2, True, False, False, True) + w.B * w.H * w.L * w.dk * 4
    row = _row(w, ms, nb, fl, peaks, peak_src, "hbm", w.B * w.L, "gdn_prefill_vector_gate")
    row["path"] = "tensor cores: vg_prep_kernel (one CTA per chunk) + vg_chain_kernel (one CTA per head)"
    rows["gdn_prefill_vector_gate"] = row
    # the same shape at head size 64 (dk = dv = 64): the one-CTA tensor-core kernel reading the
    # 64-wide tiles directly (bytes and FLOP counted at d = 64, the call's own work)
    inp64 = W.make_prefill_inputs(w.B, w.H, w.L, 64, 64, mode="gdn", in_dtype=torch.bfloat16,
                                  seed=W.SEED_BASE + 8, device="cuda")
    o64 = torch.empty(w.B, w.H, w.L, 64, device="cuda")
    sf64 = torch.empty(w.B, w.H, 64, 64, device="cuda")
    fn = lambda: gdn.gdn_chunk_fwd(inp64["q"], inp64["k"], inp64["v"], inp64["beta"], inp64["g"], o=o64,
                                   s_final=sf64, chunk=w.chunk)
    ms = timed(fn, max(5, args.steps), 3)
    nb64 = prefill_bytes(w.B, w.H, w.L, 64, 64, 2, True, True, False, True)
    fl64 = flops_per_head_token("gdn", 64, 64, w.chunk) * w.B * w.H * w.L
    row = _row(w, ms, nb64, fl64, peaks, peak_src, "hbm", w.B * w.L)
    row["workload"] = "gdn_bf16_B8_H16_L4096_d64"
    row["path"] = "tc_gdn_kernel, narrow instantiation (64-wide tensor maps; the far tile halves load as zeros)"
    rows["gdn_prefill_d64"] = row
    del inp64, o64, sf64
    del inp, o, sf, gv
    # backward pass (gradients of the prefill) on the headline shape: fp32 CUDA-core kernel whose
    # per-token state traffic goes through the caller's workspace (checkpoints + chunk slab)
    inp = W.make_workload_inputs(w, device="cuda")
    do = torch.randn(w.B, w.H, w.L, w.dv, device="cuda")
    ws = torch.empty(gdn.gdn_chunk_bwd_workspace_bytes(w.B, w.H, w.L, w.dk, w.dv, w.chunk), dtype=torch.uint8,
                     device="cuda")
    fn = lambda: gdn.gdn_chunk_bwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["g"], do, chunk=w.chunk, workspace=ws)
    ms = timed(fn, max(3, args.steps // 10), 1)
    rows["gdn_bwd"] = bwd_row(w, ms, peaks, peak_src)
    del inp, do, ws
    torch.cuda.empty_cache()
    # long-context Gated DeltaNet, 1 x 32 x 65536 x 128, S0 != 0
    w = W.WORKLOADS[3]
    inp = W.make_workload_inputs(w, device="cuda")
    o = torch.empty(w.B, w.H, w.L, w.dv, device="cuda")
    sf = torch.empty(w.B, w.H, w.dk, w.dv, device="cuda")
    fn = lambda: gdn.gdn_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["g"], o=o,
                                   s0=inp["s0"], s_final=sf, chunk=w.chunk)
    ms = timed(fn, max(10, args.steps // 2), 3)
    nb = prefill_bytes(w.B, w.H, w.L, w.dk, w.dv, 2, True, True, True, True)
    fl = flops_per_head_token("gdn", w.dk, w.dv, w.chunk) * w.B * w.H * w.L
    row = _row(w, ms, nb, fl, peaks, peak_src, "hbm", w.B * w.L, "gdn_prefill_long")
    row["path"] = ("vg_prep_kernel (all SMs) + vg_chain_kernel (one CTA per head) in 16 segments of 64 chunks; "
                   "the prep of segment i+1 overlaps the chain of segment i (two library streams)")
    rows["gdn_prefill_long"] = row
    # the same workload as a sequence split into 3 segments on this one device: segments 0-1
    # (from s0 / from 0) with segment 1 from lambda I alongside (96 one-CTA sequences, one
    # wave on 148 SMs), the composition, then segments 1-2 again from their incoming states;
    # bytes and FLOP counted as for one pass (the algorithmic work of the operator), so the
    # fraction shows what the split costs on one device
    from gated_deltanet_sequence_b200.context_parallel import segmented_prefill, segment_bounds
    bounds = segment_bounds(w.L, 3, w.chunk)
    fn = lambda: segmented_prefill(inp["q"], inp["k"], inp["v"], inp["beta"], inp["g"], inp["s0"], o=o,
                                   s_final=sf, chunk=w.chunk, bounds=bounds)
    ms = timed(fn, max(3, args.steps // 4), 2)
    row = _row(w, ms, nb, fl, peaks, peak_src, "hbm", w.B * w.L)
    row["path"] = "sequence split, 3 segments on one device (3 packed launches + 1 composition)"
    rows["gdn_prefill_long_split3"] = row
    del inp, o, sf
    torch.cuda.empty_cache()
    # packed variable-length Gated DeltaNet: 24 sequences (log-uniform length mix), 16 heads
    wv = W.VARLEN_WORKLOAD
    lens = W.draw_seqlens(wv["N"], wv["T"], seed=wv["seed"], min_len=wv["min_len"])
    inp = W.make_varlen_inputs(lens, wv["H"], 128, 128, mode="gdn", in_dtype=torch.bfloat16,
                               seed=wv["seed"], device="cuda")
    T, H, N = wv["T"], wv["H"], wv["N"]
    o = torch.empty(H, T, 128, device="cuda")
    sf = torch.empty(N, H, 128, 128, device="cuda")
    fn = lambda: gdn.gdn_chunk_fwd_varlen(inp["q"], inp["k"], inp["v"], inp["beta"], inp["cu_seqlens"],
                                          inp["g"], o=o, s_final=sf)
    ms = timed(fn, max(5, args.steps), 3)
    # per-token bytes as a (1, H, T) batch, plus one final state per (sequence, head)
    nb = prefill_bytes(1, H, T, 128, 128, 2, True, True, False, False) + N * H * 128 * 128 * 4
    fl = flops_per_head_token("gdn", 128, 128, 64) * H * T
    row = _row(w, ms, nb, fl, peaks, peak_src, "hbm", T)
    row["workload"] = wv["name"]
    row["seqlens"] = {"n": N, "min": min(lens), "max": max(lens), "total": T}
    rows["gdn_prefill_varlen"] = row
    del inp, o, sf
    torch.cuda.empty_cache()
    # decode: 256 sequences x 32 heads, 1000 consecutive steps, state in place
    w = W.WORKLOADS[4]
    steps = w.L if not args.quick else 100
    inp = W.make_workload_inputs(w, device="cuda", steps=steps)
    state = inp["state"]
    od = torch.empty(w.B, w.H, w.dv, device="cuda")
    it = [0]

    def dec():
        t = it[0] % steps
        gdn.gdn_decode_step(inp["q"][t], inp["k"][t], inp["v"][t], inp["beta"][t], inp["g"][t],
                            state, o=od)
        it[0] += 1

    ms = timed(dec, steps, 20)
    nb = decode_bytes(w.B, w.H, w.dk, w.dv, 2)
    gbs = nb / (ms * 1e-3) / 1e9
    rows["decode"] = {"workload": w.name, "us_per_step": round(ms * 1e3, 2), "steps_timed": steps,
                      "tokens_per_s": round(w.B / (ms * 1e-3), 1),
                      "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"],
                                   "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 4),
                                   "traffic": traffic_from_profiles("decode_step"), "peak_source": peak_src,
                                   "algorithmic_bytes_per_launch": nb}}
    del inp, state, od
    torch.cuda.empty_cache()
    return rows


def bwd_flops_per_head_token(dk: int, dv: int) -> float:
    """FLOPs per head-token of the backward kernel: two forward token steps (the checkpoint
    pass and the recompute: S^T k and the rank-1 update, 4 dk dv each) and the reverse step
    (q' do^T, Lambda^T k, S_{t-1} du, <Lambda, S_{t-1}>, S_t do, Lambda u: 2 dk dv each; the
    adjoint update 3 dk dv; its own forward step 4 dk dv)."""
    return (4 + 4 + 6 * 2 + 3 + 4) * dk * dv


def bwd_bytes(B, H, L, dk, dv, chunk, in_bytes=2) -> float:
    """Bytes one backward launch moves: inputs q, k, v (in_bytes), beta, g, do (fp32); outputs
    dq, dk, dv, dbeta, dg (fp32); and the workspace: every chunk checkpoint written once and read
    once, every in-chunk state written once to the slab and read once."""
    n = B * H * L
    io = n * ((2 * dk + dv) * in_bytes + 8 + dv * 4) + n * ((2 * dk + dv) * 4 + 8)
    nck = -(-L // chunk)
    state = dk * dv * 4
    wsb = B * H * (2 * nck * state + 2 * L * state)
    return float(io + wsb)


def bwd_row(w, ms, peaks, peak_src):
    fl = bwd_flops_per_head_token(w.dk, w.dv) * w.B * w.H * w.L
    nb = bwd_bytes(w.B, w.H, w.L, w.dk, w.dv, w.chunk)
    row = _row(w, ms, nb, fl, peaks, peak_src, "hbm", w.B * w.L)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    peak_f32 = sms * 128 * 2 * FP32_CLOCK_GHZ / 1e3
    tf = fl / (ms * 1e-3) / 1e12
    row["path"] = "fp32 reverse-mode kernel (CUDA cores), state traffic through the workspace"
    row["alu"] = {"achieved": round(tf, 2), "peak": round(peak_f32, 1), "unit": "TFLOP/s",
                  "frac": round(tf / peak_f32, 4), "algorithmic_flop_per_launch": fl}
    return row


def _row(w, ms, nbytes, flop, peaks, peak_src, bound, tokens, traffic_key=None):
    gbs = nbytes / (ms * 1e-3) / 1e9
    tfs = flop / (ms * 1e-3) / 1e12
    return {"workload": w.name, "ms_per_launch": round(ms, 4), "tokens_per_s": round(tokens / (ms * 1e-3), 1),
            "roofline": {"bound": bound, "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(gbs / peaks["hbm_gbs"], 4), "peak_source": peak_src,
                         "traffic": traffic_from_profiles(traffic_key) if traffic_key else None,
                         "algorithmic_bytes_per_launch": nbytes},
            "tensor": {"achieved": round(tfs, 1), "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                       "frac": round(tfs / peaks["bf16_tflops"], 4)}}


# ------------------------------------------------------------------------- oracle legs
def _oracle_sample(target_s: float):
    """Time the fp64 oracle on a bounded sample of the headline workload: whole heads
    (all 4096 tokens) of the 8 x 16 batch, as many as fit about ``target_s`` seconds."""
    import oracle
    w = W.WORKLOADS[2]
    cores = oracle.default_threads()
    probe = W.make_prefill_inputs(1, 1, w.L, w.dk, w.dv, mode="gdn", in_dtype=torch.bfloat16,
                                  seed=W.SEED_BASE + 2)
    t0 = time.perf_counter()
    oracle.recurrent_fwd(probe["q"], probe["k"], probe["v"], probe["beta"], probe["g"], None, nthreads=1)
    per_head = time.perf_counter() - t0
    nheads = int(max(1, min(w.B * w.H, round(target_s / per_head * cores))))
    inp = W.make_prefill_inputs(w.B, w.H, w.L, w.dk, w.dv, mode="gdn", in_dtype=torch.bfloat16,
                                seed=W.SEED_BASE + 2)
    flat = lambda x: x.reshape(w.B * w.H, *x.shape[2:])[:nheads]
    args = [flat(inp[n]) for n in ("q", "k", "v", "beta", "g")]
    t0 = time.perf_counter()
    oracle.recurrent_fwd(*args, None, nthreads=cores)
    dt = time.perf_counter() - t0
    head_tokens = nheads * w.L
    return {"value": round(head_tokens / w.H / dt, 1), "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{nheads} of {w.B * w.H} heads x {w.L} tokens of {w.name} (tokens = head-tokens / H)",
            "seconds": round(dt, 2)}


def cpu_baseline(target_s: float):
    return _oracle_sample(target_s)


def run_reference(args, rank, world):
    """The reference arm: the fp64 oracle, as it stands, timed on this host's cores.
    Each step is a bounded sample of the headline workload; only rank 0 runs."""
    if rank != 0:
        return None
    per_step = max(1.0, args.cpu_seconds / max(1, args.steps))
    vals, last = [], None
    for _ in range(max(1, args.steps)):
        last = _oracle_sample(per_step)
        vals.append(last["value"])
    value = statistics.median(vals)
    w = W.WORKLOADS[2]
    cb = dict(last)
    cb["value"] = value
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded; same generator and seed as the GPU arm)",
            "config": headline_config(world),
            "cpu_baseline": cb,
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ------------------------------------------------------------------------- profiling driver
def run_profile(spec: str):
    """Run one kernel a few times on one case (for an ncu capture; prints nothing timed).
    spec: gdn[:B] (GDN bf16, B x 16 x 4096 x 128), la[:B] (plain LA, B x 16 x 4096 x 128),
    decode[:N] (N x 32 heads, 3 steps), gdn_long (1 x 32 x 65536), gdnh[:H[:L]] (1 x H x L, S0 != 0:
    with 3 H within the SM count, the segmented prep + chain kernels from 128 chunks on, the
    cluster form below that), gdnvec[:B[:L]] (vector-valued gates, B x 16 x L,
    bf16: the prep and chain kernels), gdnvec32[:B[:L]] (the same in fp32: the fp32 chunk kernel)."""
    from gated_deltanet_sequence_b200 import _lib as gdn
    kind, _, arg = spec.partition(":")
    torch.cuda.set_device(0)
    if kind in ("gdn", "la"):
        B = int(arg or 4)
        w = W.WORKLOADS[2 if kind == "gdn" else 1]
        inp = W.make_prefill_inputs(B, w.H, w.L, w.dk, w.dv, mode=w.mode, in_dtype=torch.bfloat16,
                                    seed=W.SEED_BASE + w.index, device="cuda")
        o = torch.empty(B, w.H, w.L, w.dv, device="cuda")
        sf = torch.empty(B, w.H, w.dk, w.dv, device="cuda")
        for _ in range(3):
            if kind == "gdn":
                gdn.gdn_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["g"], o=o, s_final=sf)
            else:
                gdn.lin_attn_chunk_fwd(inp["q"], inp["k"], inp["v"], None, o=o, s_final=sf)
    elif kind == "gdnh":
        # B=1, H heads of L tokens, S0 != 0 (few heads: the segmented form, or the cluster form
        # below 128 chunks)
        H, _, L = arg.partition(":")
        H, L = int(H or 32), int(L or 8192)
        inp = W.make_prefill_inputs(1, H, L, 128, 128, mode="gdn", in_dtype=torch.bfloat16, s0=True,
                                    seed=W.SEED_BASE + 3, device="cuda")
        o = torch.empty(1, H, L, 128, device="cuda")
        sf = torch.empty(1, H, 128, 128, device="cuda")
        for _ in range(2):
            gdn.gdn_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["g"], o=o, s0=inp["s0"], s_final=sf)
    elif kind in ("gdnvec", "gdnvec32"):
        # vector-valued gates: B x 16 heads x L tokens, d = 128; bf16 inputs take the tensor-core
        # prep and chain kernels, fp32 inputs the fp32 chunk kernel
        B, _, L = arg.partition(":")
        B, L = int(B or 1), int(L or 1024)
        inp = W.make_prefill_inputs(B, 16, L, 128, 128, mode="gdn",
                                    in_dtype=torch.bfloat16 if kind == "gdnvec" else torch.float32,
                                    seed=W.SEED_BASE + 7, device="cuda")
        gv = W.make_gate_per_key((B, 16), L, 128, seed=W.SEED_BASE + 7, device="cuda")
        o = torch.empty(B, 16, L, 128, device="cuda")
        sf = torch.empty(B, 16, 128, 128, device="cuda")
        for _ in range(2):
            gdn.gdn_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["beta"], gv, o=o, s_final=sf)
    elif kind == "gdn_long":
        w = W.WORKLOADS[3]
        inp = W.make_workload_inputs(w, device="cuda")
        o = torch.empty(w.B, w.H, w.L, w.dv, device="cuda")
        sf = torch.empty(w.B, w.H, w.dk, w.dv, device="cuda")
        for _ in range(2):
            gdn.gdn_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["g"], o=o, s0=inp["s0"], s_final=sf)
    elif kind == "decode":
        N = int(arg or 64)
        inp = W.make_decode_inputs(N, 32, 128, 128, 3, device="cuda", seed=W.SEED_BASE + 4)
        for t in range(3):
            gdn.gdn_decode_step(inp["q"][t], inp["k"][t], inp["v"][t], inp["beta"][t], inp["g"][t], inp["state"])
    else:
        raise SystemExit(f"unknown profile case {spec}")
    torch.cuda.synchronize()
    if gdn.gdn_sync_status() != 0:
        raise SystemExit("device-side timeout")
    print(f"profile case {spec} done")


# ------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-rows", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--quick", action="store_true", help="shorter decode row (100 steps)")
    ap.add_argument("--profile", default=None,
                    help="run one kernel a few times for a profiler capture: gdn[:B] | la[:B] | decode[:N] | gdn_long")
    args = ap.parse_args()
    if args.profile:
        run_profile(args.profile)
        return
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    torch.cuda.set_device(local)
    pg = False
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        pg = True
    barrier, max_over_ranks = rank_collectives(world, torch.device("cuda", local))
    try:
        line = run_ours(args, rank, world, barrier, max_over_ranks)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if pg:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
