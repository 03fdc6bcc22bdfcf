"""Gated DeltaNet / DeltaNet prefill from host buffers, copies overlapped with compute.

The (sequence, head) recurrences are independent, so a batch can cross PCIe in groups of
sequences: while group i is computed, group i+1 is uploaded and group i-1 downloaded, on
three CUDA streams, with two device staging slots. Host-to-device and device-to-host copies
run at the same time (PCIe is full duplex), so a step costs about the larger of the two
transfers instead of their sum. Every group is one call of the library's prefill kernel,
which gives each (sequence, head) the same bits whatever the batch around it, so the result
equals one call on the whole batch. The library itself allocates nothing; the staging
buffers come from PyTorch's device allocator.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import _lib


def _pinned(name: str, t: Optional[torch.Tensor], required: bool = True):
    if t is None:
        if required:
            raise ValueError(f"{name} is required")
        return
    if t.device.type != "cpu" or not t.is_pinned():
        raise ValueError(f"{name} must be a pinned host tensor (torch.Tensor.pin_memory())")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def gdn_chunk_fwd_host(q, k, v, beta, g=None, o=None, s0=None, s_final=None, *, chunk: int = 64,
                       scale: float = 1.0, group: int = 1, device=None):
    """DeltaNet (g None) / Gated DeltaNet prefill of pinned host tensors (the dense layout of
    :func:`gated_deltanet_sequence_b200._lib.gdn_chunk_fwd`). ``group`` sequences cross PCIe
    per stage. ``o`` / ``s_final`` (pinned host, fp32) are allocated when None (``s_final``
    only when asked for with ``s_final=True``). The call is asynchronous: the current stream
    of ``device`` waits for the last copy, so synchronise it before reading the outputs.
    Returns (o, s_final)."""
    for name, t in (("q", q), ("k", k), ("v", v), ("beta", beta)):
        _pinned(name, t)
    _pinned("g", g, required=False)
    _pinned("s0", s0, required=False)
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    if o is None:
        o = torch.empty(B, H, L, dv, dtype=torch.float32, pin_memory=True)
    if s_final is True:
        s_final = torch.empty(B, H, dk, dv, dtype=torch.float32, pin_memory=True)
    _pinned("o", o)
    _pinned("s_final", s_final, required=False)
    if group < 1:
        raise ValueError("group must be >= 1")
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    main = torch.cuda.current_stream(dev)
    up, comp, down = (torch.cuda.Stream(dev) for _ in range(3))
    G = min(group, B)
    ins = [(q, q.shape[1:]), (k, k.shape[1:]), (v, v.shape[1:]), (beta, beta.shape[1:])]
    if g is not None:
        ins.append((g, g.shape[1:]))
    if s0 is not None:
        ins.append((s0, s0.shape[1:]))
    # two staging slots of G sequences each, allocated on the current stream
    slots = []
    with torch.cuda.stream(main):
        for _ in range(2):
            din = [torch.empty((G,) + tuple(shape), dtype=t.dtype, device=dev) for t, shape in ins]
            dout = torch.empty(G, H, L, dv, dtype=torch.float32, device=dev)
            dsf = torch.empty(G, H, dk, dv, dtype=torch.float32, device=dev) if s_final is not None else None
            for t in din + [dout] + ([dsf] if dsf is not None else []):
                for s in (up, comp, down):
                    t.record_stream(s)
            slots.append((din, dout, dsf))
    start = torch.cuda.Event()
    start.record(main)
    free_in = [start, start]     # slot's inputs no longer read (its last compute done)
    free_out = [start, start]    # slot's outputs copied out
    last = start
    for i, b0 in enumerate(range(0, B, G)):
        b1 = min(B, b0 + G)
        n = b1 - b0
        din, dout, dsf = slots[i % 2]
        up.wait_event(free_in[i % 2])
        with torch.cuda.stream(up):
            for d, (t, _) in zip(din, ins):
                d[:n].copy_(t[b0:b1], non_blocking=True)
            loaded = torch.cuda.Event()
            loaded.record(up)
        comp.wait_event(loaded)
        comp.wait_event(free_out[i % 2])
        with torch.cuda.stream(comp):
            dq, dk_, dv_, db = din[:4]
            dg = din[4] if g is not None else None
            ds0 = din[-1] if s0 is not None else None
            _lib.gdn_chunk_fwd(dq[:n], dk_[:n], dv_[:n], db[:n], None if dg is None else dg[:n],
                               o=dout[:n], s0=None if ds0 is None else ds0[:n],
                               s_final=None if dsf is None else dsf[:n], chunk=chunk, scale=scale, stream=comp)
            done = torch.cuda.Event()
            done.record(comp)
        free_in[i % 2] = done
        down.wait_event(done)
        with torch.cuda.stream(down):
            o[b0:b1].copy_(dout[:n], non_blocking=True)
            if s_final is not None:
                s_final[b0:b1].copy_(dsf[:n], non_blocking=True)
            out = torch.cuda.Event()
            out.record(down)
        free_out[i % 2] = out
        last = out
    main.wait_event(last)
    return o, s_final
