"""fp64 CPU oracle for chunkwise Gated DeltaNet — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its CPU-baseline
and reference legs) may import this package. It shares no code with the CUDA
library: the arithmetic lives in ``gdn_oracle.c`` (plain C, IEEE double, no
fast-math), compiled here with gcc and called through ctypes.

Functions (each cites the passages it follows in ``gdn_oracle.c``):
  recurrent_fwd  token-by-token recurrence, the definition of the operator (optionally
                 with Mamba's skip term o_t += D_h v_t, added here in numpy)
  decode_step    one token for many independent heads, state in place (scalar or
                 vector-valued gates, optional skip term)
  xnorm          the output normalisation of the "Devil in Linear Transformer" form (RMS
                 or layer normalisation of each output row over dv, with weights (H, dv))
  chunked_fwd    fp64 chunkwise re-derivation (UT/WY form) for invariance tests
  ut_transform   the per-chunk T = (I + A)^-1 factor
  recurrent_bwd  gradients of the operator (dq, dk, dv, dbeta, dg, ds0) by fp64 autograd of
                 the token recurrence written out in PyTorch CPU ops

Pins (tests/test_oracle_pins.py) tie these to what the pages fix: the masked
parallel form, the positions 1-4 cumulative-sum example, the delta rule as one
gradient step, exact key->value recall, the Householder reflection, brute-force
transition products, the WY product form and chunk-size invariance; the skip term and
the vector-valued gates have their own (tests/test_oracle_dskip.py,
tests/test_oracle_vector_gate.py).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def compile_c(src: str, out: str) -> str:
    """gcc -O2 (no fast-math, no FMA contraction) of one C file into a shared library."""
    tmp = out + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-std=c11",
                           "-fPIC", "-shared", "-o", tmp, src, "-lm", "-lpthread"])
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile gdn_oracle.c into liboracle.so when missing or stale."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        compile_c(_SRC, _LIB_PATH)
    return _LIB_PATH


def load_variant(path: str):
    """Bind a separately compiled copy of the oracle (used to plant mistakes in tests)."""
    return _bind(path)


def _bind(path: str):
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    l, d, i = ctypes.c_long, ctypes.c_double, ctypes.c_int
    lib.oracle_recurrent_fwd.argtypes = [P, P, P, P, P, P, P, P, l, l, l, l, d, i]
    lib.oracle_recurrent_fwd_vg.argtypes = [P, P, P, P, P, P, P, P, l, l, l, l, d, i]
    lib.oracle_decode_step.argtypes = [P, P, P, P, P, P, P, l, l, l, d, i]
    lib.oracle_decode_step_vg.argtypes = [P, P, P, P, P, P, P, l, l, l, d, i]
    lib.oracle_chunked_fwd.argtypes = [P, P, P, P, P, P, P, P, l, l, l, l, l, d, i]
    lib.oracle_ut_transform.argtypes = [P, P, P, P, l, l]
    for f in (lib.oracle_recurrent_fwd, lib.oracle_recurrent_fwd_vg, lib.oracle_decode_step, lib.oracle_decode_step_vg,
              lib.oracle_chunked_fwd, lib.oracle_ut_transform):
        f.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _bind(build())
    return _lib


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _f64(x) -> Optional[np.ndarray]:
    """Exact upcast of a torch tensor / array (bf16, fp32, fp64) to C-contiguous fp64."""
    if x is None:
        return None
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def xnorm(o, kind: str, weight=None, eps: float = 1e-6):
    """Output normalisation of page "LinearAttention 概述", section "The Devil in Linear
    Transformer": the normaliser's denominator is dropped and the output is normalised
    instead, O = XNorm(Q (K^T V)). The page does not fix XNorm's form; the reading taken:
    each output row o_t of each head is normalised over its dv values,
      kind "rms":   o_t / sqrt(mean_c o_t[c]^2 + eps)
      kind "layer": (o_t - mean_c o_t[c]) / sqrt(mean_c (o_t[c] - mean)^2 + eps)
    then multiplied elementwise by weight[h] (shape (H, dv); None = ones).
    o: (..., H, L, dv); returns a new float64 array."""
    o = _f64(o)
    if kind == "layer":
        x = o - o.mean(axis=-1, keepdims=True)
    elif kind == "rms":
        x = o
    else:
        raise ValueError(f"xnorm kind {kind!r}")
    out = x / np.sqrt((x * x).mean(axis=-1, keepdims=True) + eps)
    if weight is not None:
        w = _f64(weight)
        if o.ndim < 3 or w.shape != (o.shape[-3], o.shape[-1]):
            raise ValueError(f"xnorm weight: expected (H, dv), got {w.shape}")
        out = out * w[:, None, :]
    return out


def recurrent_fwd(q, k, v, beta=None, g=None, s0=None, scale: float = 1.0,
                  nthreads: Optional[int] = None, lib=None, d_skip=None):
    """Token-by-token fp64 recurrence.

    q, k: (..., H, L, dk); v: (..., H, L, dv); beta: (..., H, L) or None; g: (..., H, L)
    (one log-decay per token) or (..., H, L, dk) (vector-valued gate, one log-decay per key
    coordinate: row j of the state decays by exp(g_t[j]), the GLA-style variant next to the
    scalar gate) or None; s0: (..., H, dk, dv) or None. d_skip: (H, dv) or None, the skip term of Mamba (page
    "【CS336】lecture4", section "继续改进：Mamba": a term in v is added to the output, like
    a residual connection, so the input reaches the output without passing the state):
    o_t += d_skip[h] * v_t elementwise. Returns (o (..., H, L, dv), S_final (..., H, dk,
    dv)) as float64 arrays.
    """
    q, k, v, beta, g, s0 = map(_f64, (q, k, v, beta, g, s0))
    lead = q.shape[:-2]
    L, dk = q.shape[-2:]
    dv = v.shape[-1]
    BH = int(np.prod(lead)) if lead else 1
    o = np.zeros(lead + (L, dv), np.float64)
    sf = np.zeros(lead + (dk, dv), np.float64)
    vector_gate = g is not None and g.ndim == q.ndim
    if g is not None and g.shape != (q.shape if vector_gate else q.shape[:-1]):
        raise ValueError(f"g: expected {q.shape[:-1]} or {q.shape}, got {g.shape}")
    lib_ = lib or _load()
    fn = lib_.oracle_recurrent_fwd_vg if vector_gate else lib_.oracle_recurrent_fwd
    rc = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g), _ptr(s0), _ptr(o), _ptr(sf), BH, L, dk, dv,
            float(scale), nthreads or default_threads())
    if rc:
        raise ValueError("oracle_recurrent_fwd: bad sizes")
    if d_skip is not None:
        D = _f64(d_skip)
        if not lead or D.shape != (lead[-1], dv):
            raise ValueError(f"d_skip: expected (H, dv) = ({lead[-1] if lead else '?'}, {dv}), got {D.shape}")
        o += D.reshape((1,) * (len(lead) - 1) + (lead[-1], 1, dv)) * v
    return o, sf


def recurrent_fwd_varlen(q, k, v, cu_seqlens, beta=None, g=None, s0=None, scale: float = 1.0,
                         nthreads: Optional[int] = None, lib=None, d_skip=None):
    """Packed variable-length batch: every sequence is its own recurrence.

    q, k: (H, T, dk); v: (H, T, dv); beta, g: (H, T) or None; cu_seqlens: N + 1 offsets
    (sequence n of every head is tokens cu[n] .. cu[n+1]-1); s0: (N, H, dk, dv) or None.
    Each sequence runs through :func:`recurrent_fwd` from its own initial state. Returns
    (o (H, T, dv) with zeros at rows outside every sequence, S_final (N, H, dk, dv)).
    d_skip (H, dv) as for :func:`recurrent_fwd`.
    """
    q, k, v, beta, g, s0 = map(_f64, (q, k, v, beta, g, s0))
    cu = [int(x) for x in np.asarray(cu_seqlens).reshape(-1)]
    H, T, dk = q.shape
    dv = v.shape[-1]
    N = len(cu) - 1
    o = np.zeros((H, T, dv), np.float64)
    sf = np.zeros((N, H, dk, dv), np.float64)
    for n in range(N):
        a, b = cu[n], cu[n + 1]
        if not (0 <= a <= b <= T):
            raise ValueError(f"cu_seqlens[{n}:{n + 2}] = {a}, {b} is not a range inside [0, {T}]")
        sl = slice(a, b)
        on, sfn = recurrent_fwd(q[:, sl], k[:, sl], v[:, sl],
                                None if beta is None else beta[:, sl], None if g is None else g[:, sl],
                                None if s0 is None else s0[n], scale, nthreads, lib, d_skip)
        o[:, sl] = on
        sf[n] = sfn
    return o, sf


def decode_step(q, k, v, beta, g, state: np.ndarray, scale: float = 1.0,
                nthreads: Optional[int] = None, lib=None, d_skip=None):
    """One decode token for every head; ``state`` (fp64, (..., dk, dv)) is updated in place.

    q, k: (..., H, dk); v: (..., H, dv); beta: (..., H) or None; g: (..., H) or (..., H, dk)
    (vector-valued gate, as in :func:`recurrent_fwd`) or None; d_skip (H, dv) or None (the
    skip term of :func:`recurrent_fwd`). Returns o (..., H, dv).
    """
    q, k, v, beta, g = map(_f64, (q, k, v, beta, g))
    assert state.dtype == np.float64 and state.flags.c_contiguous
    lead = q.shape[:-1]
    dk, dv = state.shape[-2:]
    NH = int(np.prod(lead)) if lead else 1
    o = np.zeros(lead + (dv,), np.float64)
    vector_gate = g is not None and g.ndim == q.ndim
    lib_ = lib or _load()
    fn = lib_.oracle_decode_step_vg if vector_gate else lib_.oracle_decode_step
    rc = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g), _ptr(state), _ptr(o), NH, dk, dv, float(scale),
            nthreads or default_threads())
    if rc:
        raise ValueError("oracle_decode_step: bad sizes")
    if d_skip is not None:
        D = _f64(d_skip)
        if not lead or D.shape != (lead[-1], dv):
            raise ValueError(f"d_skip: expected (H, dv), got {D.shape}")
        o += D * v
    return o


def chunked_fwd(q, k, v, beta=None, g=None, s0=None, chunk: int = 64, scale: float = 1.0,
                nthreads: Optional[int] = None, lib=None):
    """fp64 chunkwise (UT/WY) form; same contract as :func:`recurrent_fwd`."""
    q, k, v, beta, g, s0 = map(_f64, (q, k, v, beta, g, s0))
    lead = q.shape[:-2]
    L, dk = q.shape[-2:]
    dv = v.shape[-1]
    BH = int(np.prod(lead)) if lead else 1
    o = np.zeros(lead + (L, dv), np.float64)
    sf = np.zeros(lead + (dk, dv), np.float64)
    rc = (lib or _load()).oracle_chunked_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g), _ptr(s0),
                                    _ptr(o), _ptr(sf), BH, L, dk, dv, int(chunk), float(scale),
                                    nthreads or default_threads())
    if rc:
        raise ValueError("oracle_chunked_fwd: bad sizes")
    return o, sf


def ut_transform(K, beta, g=None, lib=None):
    """T = (I + A)^-1 for one chunk (K: n x dk, beta: n, g: n or None)."""
    K, beta, g = map(_f64, (K, beta, g))
    n, dk = K.shape
    T = np.zeros((n, n), np.float64)
    rc = (lib or _load()).oracle_ut_transform(_ptr(K), _ptr(beta), _ptr(g), _ptr(T), n, dk)
    if rc:
        raise ValueError("oracle_ut_transform: bad sizes")
    return T


def recurrent_bwd(q, k, v, beta=None, g=None, s0=None, do=None, ds_final=None, scale: float = 1.0):
    """Gradients of the operator (page "混合注意力学习(1)", section "Transformers 就是 RNNs":
    on the full training sequence every gradient follows from the chain rule through the
    recurrence; the page's formulas are stripped, so the reading is the exact gradient of
    the definition). The token recurrence of :func:`recurrent_fwd` (read, blend, write,
    then read out) written out in fp64 PyTorch CPU ops and differentiated by autograd, for
    the loss sum(o * do) + sum(S_final * ds_final).

    q, k: (..., L, dk); v, do: (..., L, dv); beta, g: (..., L) or None; s0, ds_final:
    (..., dk, dv) or None. Returns (o, S_final, grads) with grads a dict of float64 arrays:
    dq, dk, dv, dbeta (or None), dg (or None), ds0 (zeros when s0 is None)."""
    import torch
    t = lambda x: None if x is None else torch.tensor(_f64(x), dtype=torch.float64, requires_grad=True)
    q_, k_, v_, b_, g_ = map(t, (q, k, v, beta, g))
    lead = q_.shape[:-2]
    L, dk = q_.shape[-2:]
    dv = v_.shape[-1]
    s0_ = t(s0) if s0 is not None else torch.zeros(lead + (dk, dv), dtype=torch.float64, requires_grad=True)
    S = s0_
    outs = []
    for i in range(L):
        kt, vt = k_[..., i, :], v_[..., i, :]
        alpha = torch.exp(g_[..., i]) if g_ is not None else torch.ones(lead, dtype=torch.float64)
        if b_ is not None:
            read = torch.einsum("...jc,...j->...c", S, kt)                  # S^T k
            u = b_[..., i, None] * (vt - alpha[..., None] * read)
        else:
            u = vt
        S = alpha[..., None, None] * S + kt[..., :, None] * u[..., None, :]
        outs.append(torch.einsum("...jc,...j->...c", S, scale * q_[..., i, :]))
    o = torch.stack(outs, -2) if L else torch.zeros(lead + (0, dv), dtype=torch.float64)
    loss = (o * torch.tensor(_f64(do))).sum() if do is not None else o.sum() * 0
    if ds_final is not None:
        loss = loss + (S * torch.tensor(_f64(ds_final))).sum()
    loss.backward()
    grad = lambda x: None if x is None else (x.grad.numpy().copy() if x.grad is not None else np.zeros(x.shape))
    grads = {"dq": grad(q_), "dk": grad(k_), "dv": grad(v_), "dbeta": grad(b_), "dg": grad(g_), "ds0": grad(s0_)}
    return o.detach().numpy(), S.detach().numpy(), grads


def max_norm_err(x, ref) -> float:
    """max|x - ref| / max|ref| over the whole tensor (0 when both are all-zero)."""
    x = _f64(x)
    ref = _f64(ref)
    den = float(np.max(np.abs(ref))) if ref.size else 0.0
    num = float(np.max(np.abs(x - ref))) if ref.size else 0.0
    if den == 0.0:
        return num
    return num / den
