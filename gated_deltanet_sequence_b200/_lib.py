"""ctypes binding of libgdn.so (the C ABI declared in include/gdn.h).

Argument marshalling only: tensors are checked for dtype, shape, device and
contiguity, their data pointers and sizes are passed to the C entry points, and a
non-OK status raises. Every step of the computation runs in the library's CUDA
kernels; there is no other code path. The library must be built
(``python -m gated_deltanet_sequence_b200.build``); if it is missing, importing this
module raises ImportError. With GDN_LIBRARY=debug in the environment the bounds-checked
build (libgdn_debug.so, ``build --debug-bounds``) is loaded instead.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgdn_debug.so" if os.environ.get("GDN_LIBRARY") == "debug" else "libgdn.so")

GDN_OK, GDN_ERR_INVALID_ARG, GDN_ERR_UNSUPPORTED, GDN_ERR_CUDA, GDN_ERR_TIMEOUT, GDN_ERR_NONFINITE, GDN_ERR_BOUNDS = range(7)
GDN_F32, GDN_BF16 = 0, 1

EXPORTS = ("lin_attn_chunk_fwd", "gdn_chunk_fwd", "lin_attn_chunk_fwd_varlen", "gdn_chunk_fwd_varlen",
           "lin_attn_chunk_fwd_ex", "gdn_chunk_fwd_ex", "gdn_decode_step", "gdn_decode_step_ex",
           "gdn_status_str", "gdn_sync_status", "gdn_set_wait_limit_for_testing", "gdn_version",
           "gdn_chunk_bwd", "gdn_chunk_bwd_workspace_bytes", "gdn_chunk_bwd_noalloc", "gdn_state_compose",
           "gdn_state_identity", "gdn_chunk_fwd_host", "gdn_chunk_fwd_host_staging_bytes")


GDN_XNORM = {None: 0, "rms": 1, "layer": 2}


class FwdOpts(ctypes.Structure):
    """gdn_fwd_opts_t: dtype of o, the D-skip weights (H, dv) (device pointer or None), the
    vector-valued gate flag (g holds one log-decay per key coordinate) and the output
    normalisation (kind, weights (H, dv) or None, eps)."""
    _fields_ = [("out_dtype", ctypes.c_int), ("d_skip", ctypes.c_void_p), ("g_per_key", ctypes.c_int),
                ("xnorm", ctypes.c_int), ("xnorm_weight", ctypes.c_void_p), ("xnorm_eps", ctypes.c_float)]


class GdnError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {status_str(status)} ({status})")
        self.status = status


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{os.path.basename(LIB_PATH)} is not built ({LIB_PATH}); run "
                          "`python -m gated_deltanet_sequence_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.lin_attn_chunk_fwd.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, F, I, P]
    lib.gdn_chunk_fwd.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, F, I, P]
    lib.lin_attn_chunk_fwd_varlen.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, F, I, P]
    lib.gdn_chunk_fwd_varlen.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, F, I, P]
    lib.lin_attn_chunk_fwd_ex.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, F, I, P, P]
    lib.gdn_chunk_fwd_ex.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, F, I, P, P]
    lib.gdn_decode_step.argtypes = [P, P, P, P, P, P, P, I, I, I, I, F, I, P]
    lib.gdn_decode_step_ex.argtypes = [P, P, P, P, P, P, P, I, I, I, I, F, I, P, P]
    lib.gdn_status_str.argtypes = [I]
    lib.gdn_status_str.restype = ctypes.c_char_p
    lib.gdn_sync_status.argtypes = [P]
    lib.gdn_version.argtypes = []
    lib.gdn_set_wait_limit_for_testing.argtypes = [ctypes.c_longlong]
    Z = ctypes.c_size_t
    lib.gdn_chunk_bwd_workspace_bytes.argtypes = [I, I, I, I, I, I]
    lib.gdn_chunk_bwd_workspace_bytes.restype = Z
    lib.gdn_chunk_bwd.argtypes = [P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, Z, I, I, I, I, I, I, F, I, P]
    lib.gdn_chunk_bwd.restype = ctypes.c_int
    lib.gdn_chunk_bwd_noalloc.argtypes = [P, P, P, P, P, P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, F, I, P]
    lib.gdn_chunk_bwd_noalloc.restype = ctypes.c_int
    lib.gdn_set_wait_limit_for_testing.restype = None
    lib.gdn_state_compose.argtypes = [P, P, P, P, F, I, I, P]
    lib.gdn_state_compose.restype = ctypes.c_int
    lib.gdn_state_identity.argtypes = [P, F, I, I, P]
    lib.gdn_chunk_fwd_host_staging_bytes.argtypes = [I, I, I, I, I, I, I, I, I, I]
    lib.gdn_chunk_fwd_host_staging_bytes.restype = Z
    lib.gdn_chunk_fwd_host.argtypes = [P, P, P, P, P, P, P, P, P, Z, I, I, I, I, I, I, F, I, I, P]
    lib.gdn_chunk_fwd_host.restype = ctypes.c_int
    lib.gdn_state_identity.restype = ctypes.c_int
    for f in (lib.lin_attn_chunk_fwd, lib.gdn_chunk_fwd, lib.lin_attn_chunk_fwd_varlen,
              lib.gdn_chunk_fwd_varlen, lib.lin_attn_chunk_fwd_ex, lib.gdn_chunk_fwd_ex,
              lib.gdn_decode_step, lib.gdn_decode_step_ex, lib.gdn_sync_status, lib.gdn_version):
        f.restype = ctypes.c_int
    return lib


lib = _load()


def status_str(status: int) -> str:
    return lib.gdn_status_str(int(status)).decode()


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return GDN_BF16
    if t.dtype == torch.float32:
        return GDN_F32
    raise TypeError(f"q/k/v must be bfloat16 or float32, got {t.dtype}")


def _check(name: str, t: Optional[torch.Tensor], shape, dtype=None, device=None, required=True):
    if t is None:
        if required:
            raise ValueError(f"{name} is required")
        return
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if device is not None and t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")


def _raise(fn: str, st: int):
    if st != GDN_OK:
        raise GdnError(fn, st)


def _check_gate(g, tok_shape, dk, dev):
    """g is one log-decay per token (tok_shape) or per token and key coordinate
    (tok_shape + (dk,), a vector-valued gate); returns whether it is the latter."""
    if g is None:
        return False
    vec = g.dim() == len(tok_shape) + 1
    _check("g", g, tuple(tok_shape) + ((dk,) if vec else ()), torch.float32, dev)
    return vec


def _out_opts(o, out_dtype, d_skip, H, dv, dev, g_per_key=False, xnorm=None, xnorm_weight=None, xnorm_eps=1e-6):
    """Output dtype (from ``o`` when given, else ``out_dtype``, default fp32), the checked
    D-skip weights, the vector-gate flag and the output normalisation (xnorm None, "rms" or
    "layer"; xnorm_weight (H, dv) fp32 or None; xnorm_eps); returns (dtype, FwdOpts or None
    when all are defaults)."""
    dt = o.dtype if o is not None else (out_dtype or torch.float32)
    if dt not in (torch.float32, torch.bfloat16):
        raise TypeError(f"o / out_dtype must be float32 or bfloat16, got {dt}")
    _check("d_skip", d_skip, (H, dv), torch.float32, dev, required=False)
    if xnorm not in GDN_XNORM:
        raise ValueError(f"xnorm must be None, 'rms' or 'layer', got {xnorm!r}")
    _check("xnorm_weight", xnorm_weight, (H, dv), torch.float32, dev, required=False)
    if xnorm is None and xnorm_weight is not None:
        raise ValueError("xnorm_weight given without xnorm")
    if dt == torch.float32 and d_skip is None and not g_per_key and xnorm is None:
        return dt, None
    return dt, FwdOpts(GDN_BF16 if dt == torch.bfloat16 else GDN_F32,
                       None if d_skip is None else d_skip.data_ptr(), int(bool(g_per_key)), GDN_XNORM[xnorm],
                       None if xnorm_weight is None else xnorm_weight.data_ptr(), float(xnorm_eps))


def lin_attn_chunk_fwd(q, k, v, g=None, o=None, s0=None, s_final=None, chunk: int = 64,
                       scale: float = 1.0, stream=None, out_dtype=None, d_skip=None, xnorm=None,
                       xnorm_weight=None, xnorm_eps: float = 1e-6):
    """Plain (g None) or gated causal linear attention. Returns (o, s_final).

    out_dtype (torch.float32 / torch.bfloat16) sets the dtype of a new ``o``; d_skip (H, dv)
    fp32 adds the skip term o_t += d_skip[h] * v_t. g of shape (B, H, L, dk) is a
    vector-valued gate (row j of the state decays by exp(g_t[j])); it runs on the fp32
    chunk kernel. xnorm ("rms" / "layer"), xnorm_weight (H, dv) and xnorm_eps normalise each
    output row over dv after the skip term (the output normalisation of the options)."""
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    _check("q", q, (B, H, L, dk), device=dev)
    _check("k", k, (B, H, L, dk), q.dtype, dev)
    _check("v", v, (B, H, L, dv), q.dtype, dev)
    vec = _check_gate(g, (B, H, L), dk, dev)
    _check("s0", s0, (B, H, dk, dv), torch.float32, dev, required=False)
    odt, opts = _out_opts(o, out_dtype, d_skip, H, dv, dev, vec, xnorm, xnorm_weight, xnorm_eps)
    if o is None:
        o = torch.empty(B, H, L, dv, dtype=odt, device=dev)
    _check("o", o, (B, H, L, dv), odt, dev)
    _check("s_final", s_final, (B, H, dk, dv), torch.float32, dev, required=False)
    if opts is None:
        st = lib.lin_attn_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(o), _ptr(s0),
                                    _ptr(s_final), B, H, L, dk, dv, int(chunk), float(scale),
                                    _dtype_code(q), _stream(stream))
        _raise("lin_attn_chunk_fwd", st)
    else:
        st = lib.lin_attn_chunk_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(o), _ptr(s0),
                                       _ptr(s_final), None, B, H, L, dk, dv, int(chunk), float(scale),
                                       _dtype_code(q), ctypes.byref(opts), _stream(stream))
        _raise("lin_attn_chunk_fwd_ex", st)
    return o, s_final


def gdn_chunk_fwd(q, k, v, beta, g=None, o=None, s0=None, s_final=None, chunk: int = 64,
                  scale: float = 1.0, stream=None, out_dtype=None, d_skip=None, xnorm=None,
                  xnorm_weight=None, xnorm_eps: float = 1e-6):
    """DeltaNet (g None) or Gated DeltaNet chunkwise prefill. Returns (o, s_final).
    out_dtype, d_skip and the xnorm options as for :func:`lin_attn_chunk_fwd`."""
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    _check("q", q, (B, H, L, dk), device=dev)
    _check("k", k, (B, H, L, dk), q.dtype, dev)
    _check("v", v, (B, H, L, dv), q.dtype, dev)
    _check("beta", beta, (B, H, L), torch.float32, dev, required=L > 0)
    vec = _check_gate(g, (B, H, L), dk, dev)
    _check("s0", s0, (B, H, dk, dv), torch.float32, dev, required=False)
    odt, opts = _out_opts(o, out_dtype, d_skip, H, dv, dev, vec, xnorm, xnorm_weight, xnorm_eps)
    if o is None:
        o = torch.empty(B, H, L, dv, dtype=odt, device=dev)
    _check("o", o, (B, H, L, dv), odt, dev)
    _check("s_final", s_final, (B, H, dk, dv), torch.float32, dev, required=False)
    if opts is None:
        st = lib.gdn_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g), _ptr(o), _ptr(s0),
                               _ptr(s_final), B, H, L, dk, dv, int(chunk), float(scale),
                               _dtype_code(q), _stream(stream))
        _raise("gdn_chunk_fwd", st)
    else:
        st = lib.gdn_chunk_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g), _ptr(o), _ptr(s0),
                                  _ptr(s_final), None, B, H, L, dk, dv, int(chunk), float(scale),
                                  _dtype_code(q), ctypes.byref(opts), _stream(stream))
        _raise("gdn_chunk_fwd_ex", st)
    return o, s_final


def _check_varlen(q, k, v, cu_seqlens, s0, s_final):
    if q.dim() != 3:
        raise ValueError(f"q: expected (H, T, dk), got shape {tuple(q.shape)}")
    H, T, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    _check("q", q, (H, T, dk), device=dev)
    _check("k", k, (H, T, dk), q.dtype, dev)
    _check("v", v, (H, T, dv), q.dtype, dev)
    if cu_seqlens.dim() != 1 or cu_seqlens.numel() < 2:
        raise ValueError("cu_seqlens: expected (N + 1,) with N >= 1")
    _check("cu_seqlens", cu_seqlens, (cu_seqlens.numel(),), torch.int32, dev)
    N = cu_seqlens.numel() - 1
    _check("s0", s0, (N, H, dk, dv), torch.float32, dev, required=False)
    _check("s_final", s_final, (N, H, dk, dv), torch.float32, dev, required=False)
    return N, H, T, dk, dv, dev


def lin_attn_chunk_fwd_varlen(q, k, v, cu_seqlens, g=None, o=None, s0=None, s_final=None,
                              chunk: int = 64, scale: float = 1.0, stream=None, out_dtype=None,
                              d_skip=None, xnorm=None, xnorm_weight=None, xnorm_eps: float = 1e-6):
    """Packed variable-length batch of plain / gated linear attention.

    q, k (H, T, dk); v (H, T, dv); g (H, T) or None; cu_seqlens (N + 1,) int32 on the device
    (sequence n is tokens cu[n] .. cu[n+1]-1 of every head). s0, s_final (N, H, dk, dv).
    Returns (o, s_final); rows outside every sequence are left as they were in ``o``.
    out_dtype, d_skip and the xnorm options as for :func:`lin_attn_chunk_fwd`."""
    N, H, T, dk, dv, dev = _check_varlen(q, k, v, cu_seqlens, s0, s_final)
    vec = _check_gate(g, (H, T), dk, dev)
    odt, opts = _out_opts(o, out_dtype, d_skip, H, dv, dev, vec, xnorm, xnorm_weight, xnorm_eps)
    if o is None:
        o = torch.zeros(H, T, dv, dtype=odt, device=dev)
    _check("o", o, (H, T, dv), odt, dev)
    if opts is None:
        st = lib.lin_attn_chunk_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(o), _ptr(s0),
                                           _ptr(s_final), _ptr(cu_seqlens), N, H, T, dk, dv, int(chunk),
                                           float(scale), _dtype_code(q), _stream(stream))
        _raise("lin_attn_chunk_fwd_varlen", st)
    else:
        st = lib.lin_attn_chunk_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(o), _ptr(s0),
                                       _ptr(s_final), _ptr(cu_seqlens), N, H, T, dk, dv, int(chunk),
                                       float(scale), _dtype_code(q), ctypes.byref(opts), _stream(stream))
        _raise("lin_attn_chunk_fwd_ex", st)
    return o, s_final


def gdn_chunk_fwd_varlen(q, k, v, beta, cu_seqlens, g=None, o=None, s0=None, s_final=None,
                         chunk: int = 64, scale: float = 1.0, stream=None, out_dtype=None, d_skip=None,
                         xnorm=None, xnorm_weight=None, xnorm_eps: float = 1e-6):
    """Packed variable-length batch of DeltaNet / Gated DeltaNet (see lin_attn_chunk_fwd_varlen);
    beta (H, T) fp32."""
    N, H, T, dk, dv, dev = _check_varlen(q, k, v, cu_seqlens, s0, s_final)
    _check("beta", beta, (H, T), torch.float32, dev, required=T > 0)
    vec = _check_gate(g, (H, T), dk, dev)
    odt, opts = _out_opts(o, out_dtype, d_skip, H, dv, dev, vec, xnorm, xnorm_weight, xnorm_eps)
    if o is None:
        o = torch.zeros(H, T, dv, dtype=odt, device=dev)
    _check("o", o, (H, T, dv), odt, dev)
    if opts is None:
        st = lib.gdn_chunk_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g), _ptr(o), _ptr(s0),
                                      _ptr(s_final), _ptr(cu_seqlens), N, H, T, dk, dv, int(chunk),
                                      float(scale), _dtype_code(q), _stream(stream))
        _raise("gdn_chunk_fwd_varlen", st)
    else:
        st = lib.gdn_chunk_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g), _ptr(o), _ptr(s0),
                                  _ptr(s_final), _ptr(cu_seqlens), N, H, T, dk, dv, int(chunk),
                                  float(scale), _dtype_code(q), ctypes.byref(opts), _stream(stream))
        _raise("gdn_chunk_fwd_ex", st)
    return o, s_final


def gdn_decode_step(q, k, v, beta, g, state, o=None, scale: float = 1.0, stream=None, out_dtype=None,
                    d_skip=None, xnorm=None, xnorm_weight=None, xnorm_eps: float = 1e-6):
    """One decode token for (N, H) heads; ``state`` (N, H, dk, dv) fp32 is updated in place.
    g (N, H) or (N, H, dk) (vector-valued gate); out_dtype, d_skip and the xnorm options as
    for the prefill calls."""
    N, H, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    _check("q", q, (N, H, dk), device=dev)
    _check("k", k, (N, H, dk), q.dtype, dev)
    _check("v", v, (N, H, dv), q.dtype, dev)
    _check("beta", beta, (N, H), torch.float32, dev, required=False)
    vec = _check_gate(g, (N, H), dk, dev)
    _check("state", state, (N, H, dk, dv), torch.float32, dev)
    odt, opts = _out_opts(o, out_dtype, d_skip, H, dv, dev, vec, xnorm, xnorm_weight, xnorm_eps)
    if o is None:
        o = torch.empty(N, H, dv, dtype=odt, device=dev)
    _check("o", o, (N, H, dv), odt, dev)
    if opts is None:
        st = lib.gdn_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g), _ptr(state),
                                 _ptr(o), N, H, dk, dv, float(scale), _dtype_code(q), _stream(stream))
        _raise("gdn_decode_step", st)
    else:
        st = lib.gdn_decode_step_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g), _ptr(state),
                                    _ptr(o), N, H, dk, dv, float(scale), _dtype_code(q), ctypes.byref(opts),
                                    _stream(stream))
        _raise("gdn_decode_step_ex", st)
    return o


def gdn_sync_status(stream=None) -> int:
    """Synchronise the stream; report and clear one pending device-side condition
    (GDN_ERR_INVALID_ARG first, then GDN_ERR_TIMEOUT; GDN_OK when none is pending)."""
    return lib.gdn_sync_status(_stream(stream))


def gdn_set_wait_limit_for_testing(cycles: int) -> None:
    """Tests of the failure path only: bounded-wait limit (clock cycles) of the tensor-core
    kernels launched afterwards; cycles <= 0 restores the default (about 2 s)."""
    lib.gdn_set_wait_limit_for_testing(int(cycles))


def gdn_version() -> int:
    return lib.gdn_version()


def gdn_chunk_bwd(q, k, v, beta, g, d_o, s0=None, ds_final=None, chunk: int = 64, scale: float = 1.0,
                  workspace=None, stream=None):
    """Gradients of the prefill (beta None: linear attention) for the loss sum(o * d_o) +
    sum(S_final * ds_final). Returns a dict of fp32 tensors dq, dk, dv, dbeta (None without
    beta), dg (None without g), ds0. ``workspace``: a device tensor of at least
    gdn_chunk_bwd_workspace_bytes(...) bytes (allocated here with torch when None)."""
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    _check("q", q, (B, H, L, dk), device=dev)
    _check("k", k, (B, H, L, dk), q.dtype, dev)
    _check("v", v, (B, H, L, dv), q.dtype, dev)
    _check("beta", beta, (B, H, L), torch.float32, dev, required=False)
    _check("g", g, (B, H, L), torch.float32, dev, required=False)
    _check("d_o", d_o, (B, H, L, dv), torch.float32, dev)
    _check("s0", s0, (B, H, dk, dv), torch.float32, dev, required=False)
    _check("ds_final", ds_final, (B, H, dk, dv), torch.float32, dev, required=False)
    need = gdn_chunk_bwd_workspace_bytes(B, H, L, dk, dv, chunk)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    f32 = dict(dtype=torch.float32, device=dev)
    out = {"dq": torch.empty(B, H, L, dk, **f32), "dk": torch.empty(B, H, L, dk, **f32),
           "dv": torch.empty(B, H, L, dv, **f32), "dbeta": None if beta is None else torch.empty(B, H, L, **f32),
           "dg": None if g is None else torch.empty(B, H, L, **f32), "ds0": torch.empty(B, H, dk, dv, **f32)}
    st = lib.gdn_chunk_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g), _ptr(s0), _ptr(d_o), _ptr(ds_final),
                           _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dbeta"]), _ptr(out["dg"]),
                           _ptr(out["ds0"]), _ptr(workspace), workspace.numel() * workspace.element_size(), B, H, L,
                           dk, dv, int(chunk), float(scale), _dtype_code(q), _stream(stream))
    _raise("gdn_chunk_bwd", st)
    return out


def gdn_chunk_bwd_workspace_bytes(B: int, H: int, L: int, dk: int, dv: int, chunk: int = 64) -> int:
    """Bytes of device workspace gdn_chunk_bwd needs (0 for unsupported sizes)."""
    return int(lib.gdn_chunk_bwd_workspace_bytes(B, H, L, dk, dv, chunk))


def _states(name, t, required=True):
    """A batch of square fp32 states (..., d, d) on a CUDA device; returns (count, d)."""
    if t is None:
        if required:
            raise ValueError(f"{name} is required")
        return None
    if t.dim() < 2 or t.shape[-1] != t.shape[-2]:
        raise ValueError(f"{name}: expected (..., d, d), got {tuple(t.shape)}")
    _check(name, t, tuple(t.shape), torch.float32)
    d = t.shape[-1]
    return t.numel() // (d * d) if d else 0, d


def gdn_state_compose(mn, n, s_in, out, lam: float = 1.0, stream=None):
    """out = ((lam M + N) - N) / lam s_in + N for a batch of d x d states (the composition step
    of the sequence-split prefill: mn the end states of runs from lam * I, n those from 0;
    s_in None: out = N). mn, n, s_in, out: same shape (..., d, d) fp32 on one device; out must
    not overlap the others. Returns out."""
    count, d = _states("out", out)
    _check("mn", mn, tuple(out.shape), torch.float32, out.device)
    _check("n", n, tuple(out.shape), torch.float32, out.device)
    _check("s_in", s_in, tuple(out.shape), torch.float32, out.device, required=False)
    st = lib.gdn_state_compose(_ptr(mn), _ptr(n), _ptr(s_in), _ptr(out), float(lam), count, d, _stream(stream))
    _raise("gdn_state_compose", st)
    return out


def gdn_state_identity(s, value: float = 1.0, stream=None):
    """Write value * I into every d x d state of ``s`` ((..., d, d) fp32). Returns s."""
    count, d = _states("s", s)
    st = lib.gdn_state_identity(_ptr(s), float(value), count, d, _stream(stream))
    _raise("gdn_state_identity", st)
    return s
