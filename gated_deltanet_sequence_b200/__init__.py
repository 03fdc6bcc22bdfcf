"""B200-native chunkwise Gated DeltaNet: plain / gated linear attention, DeltaNet and
Gated DeltaNet prefill, and the recurrent decode step, as hand-written sm_100a CUDA
kernels behind a C ABI (include/gdn.h, libgdn.so).

The entry points (same names as the C ABI) load the library on first use:
    lin_attn_chunk_fwd, gdn_chunk_fwd, gdn_decode_step, gdn_sync_status, gdn_version
``workloads`` holds the seeded synthetic input generators.
"""
import importlib

_API = ("lin_attn_chunk_fwd", "gdn_chunk_fwd", "gdn_decode_step", "gdn_sync_status",
        "gdn_version", "status_str", "GdnError")

__all__ = list(_API)


def __getattr__(name):
    if name in _API:
        return getattr(importlib.import_module(__name__ + "._lib"), name)
    raise AttributeError(name)
