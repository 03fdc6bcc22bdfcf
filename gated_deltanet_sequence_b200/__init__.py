"""B200-native chunkwise Gated DeltaNet: plain / gated linear attention, DeltaNet and
Gated DeltaNet prefill, and the recurrent decode step, as hand-written sm_100a CUDA
kernels behind a C ABI (include/gdn.h, libgdn.so).

The entry points (same names as the C ABI) load the library on first use:
    lin_attn_chunk_fwd, gdn_chunk_fwd (dense batches; options out_dtype, d_skip and
    vector-valued gates through the shape of g), lin_attn_chunk_fwd_varlen,
    gdn_chunk_fwd_varlen (packed batches), gdn_decode_step, gdn_sync_status, gdn_version;
    gdn_chunk_fwd_host (module ``host``): prefill from pinned host buffers with the copies
    overlapped with compute.
``workloads`` holds the seeded synthetic input generators.
"""
import importlib

_API = ("lin_attn_chunk_fwd", "gdn_chunk_fwd", "lin_attn_chunk_fwd_varlen", "gdn_chunk_fwd_varlen",
        "gdn_decode_step", "gdn_sync_status", "gdn_version", "status_str", "GdnError")
_HOST = ("gdn_chunk_fwd_host",)

__all__ = list(_API + _HOST)


def __getattr__(name):
    if name in _API:
        return getattr(importlib.import_module(__name__ + "._lib"), name)
    if name in _HOST:
        return getattr(importlib.import_module(__name__ + ".host"), name)
    raise AttributeError(name)
