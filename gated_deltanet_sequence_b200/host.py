"""Gated DeltaNet / DeltaNet prefill from host buffers, copies overlapped with compute.

A thin binding of the library's gdn_chunk_fwd_host (include/gdn.h): the batch crosses PCIe
in groups of sequences while earlier groups are computed, on three CUDA streams the call
creates, with two device staging slots in a caller-owned buffer (allocated here with
PyTorch when not given). Every group is one dense prefill, and the (sequence, head)
recurrences are independent, so the result equals one call on the whole batch.
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
                       scale: float = 1.0, group: int = 1, device=None, staging: Optional[torch.Tensor] = None):
    """DeltaNet (g None) / Gated DeltaNet prefill of pinned host tensors (the dense layout of
    :func:`gated_deltanet_sequence_b200._lib.gdn_chunk_fwd`). ``group`` sequences cross PCIe
    per stage. ``o`` / ``s_final`` (pinned host, fp32) are allocated when None (``s_final``
    only when asked for with ``s_final=True``). ``staging``: a device uint8 buffer of at least
    gdn_chunk_fwd_host_staging_bytes bytes (allocated when None). The call is asynchronous: the
    current stream of ``device`` waits for the last copy, so synchronise it before reading the
    outputs. Returns (o, s_final)."""
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
    dt = _lib._dtype_code(q)
    need = int(_lib.lib.gdn_chunk_fwd_host_staging_bytes(B, H, L, dk, dv, int(group), dt, int(g is not None),
                                                          int(s0 is not None), int(s_final is not None)))
    if staging is None:
        staging = torch.empty(need, dtype=torch.uint8, device=dev)
    if staging.device != dev or staging.dtype != torch.uint8 or staging.numel() < need or not staging.is_contiguous():
        raise ValueError(f"staging must be a contiguous uint8 tensor of at least {need} bytes on {dev}")
    stream = torch.cuda.current_stream(dev)
    st = _lib.lib.gdn_chunk_fwd_host(_lib._ptr(q), _lib._ptr(k), _lib._ptr(v), _lib._ptr(beta), _lib._ptr(g),
                                     _lib._ptr(o), _lib._ptr(s0), _lib._ptr(s_final), _lib._ptr(staging),
                                     staging.numel(), B, H, L, dk, dv, int(chunk), float(scale), dt, int(group),
                                     _lib._stream(stream))
    _lib._raise("gdn_chunk_fwd_host", st)
    return o, s_final
