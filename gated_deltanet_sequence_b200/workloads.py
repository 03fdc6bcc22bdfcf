"""Seeded synthetic workloads for the chunkwise Gated DeltaNet operator.

This module only draws random inputs with the shapes and value distributions of
the five standard workloads. It holds none of the operator's arithmetic, so both
the CUDA path (through the binding) and the fp64 oracle under ``oracle/`` can be
fed from it without sharing any computation.

Distributions (per the workload statements):
  * q, k ~ N(0, 1), L2-normalised per head-token in fp32, then cast;
  * v ~ N(0, 1) (GDN) or N(0, 1)/sqrt(d) for q, k, v (plain linear attention);
  * beta = sigmoid(N(0, 1)) in fp32; log-alpha g ~ U(-0.05, 0) in fp32;
  * initial state S0 ~ N(0, 0.01), read as variance 0.01 (std 0.1), fp32,
    stored (dk, dv) per head.

Layouts: q, k (B, H, L, dk); v (B, H, L, dv); beta, g (B, H, L);
S (B, H, dk, dv). Decode inputs are stacked per step: (steps, N, H, d).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

SEED_BASE = 1000


@dataclasses.dataclass(frozen=True)
class Workload:
    """One standard workload: sizes, mode and input dtype."""
    index: int
    name: str
    mode: str            # "gdn" (delta + gate), "la" (plain), "decode"
    B: int
    H: int
    L: int               # sequence length (decode: number of steps)
    dk: int
    dv: int
    chunk: int
    in_dtype: torch.dtype
    s0: bool             # nonzero initial state


WORKLOADS = (
    Workload(0, "gdn_fp32_B1_H2_L256_d64", "gdn", 1, 2, 256, 64, 64, 64, torch.float32, False),
    Workload(1, "la_bf16_B4_H16_L4096_d128", "la", 4, 16, 4096, 128, 128, 64, torch.bfloat16, False),
    Workload(2, "gdn_bf16_B8_H16_L4096_d128", "gdn", 8, 16, 4096, 128, 128, 64, torch.bfloat16, False),
    Workload(3, "gdn_bf16_B1_H32_L65536_d128_s0", "gdn", 1, 32, 65536, 128, 128, 64, torch.bfloat16, True),
    Workload(4, "decode_bf16_N256_H32_d128_1000steps", "decode", 256, 32, 1000, 128, 128, 1, torch.bfloat16, True),
)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _l2norm(x: torch.Tensor) -> torch.Tensor:
    # input distribution only: unit-norm rows in fp32 before the cast
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-12)


def make_prefill_inputs(B: int, H: int, L: int, dk: int, dv: int, *, mode: str = "gdn",
                        in_dtype: torch.dtype = torch.bfloat16, s0: bool = False,
                        seed: int = SEED_BASE, device="cpu", gated: Optional[bool] = None,
                        g_low: float = -0.05) -> dict:
    """Draw one prefill batch.

    mode "gdn": q, k unit-norm, v ~ N(0,1), beta = sigmoid(N(0,1)), g ~ U(g_low, 0).
    mode "la":  q, k, v ~ N(0,1)/sqrt(dk); beta is None; g is None unless ``gated``.
    Returns a dict with q, k, v (in_dtype), beta, g, s0 (fp32 or None).
    """
    gen = _gen(seed, device)
    f32 = dict(dtype=torch.float32, device=device, generator=gen)
    q = torch.randn(B, H, L, dk, **f32)
    k = torch.randn(B, H, L, dk, **f32)
    v = torch.randn(B, H, L, dv, **f32)
    beta = g = None
    if mode == "gdn":
        q = _l2norm(q)
        k = _l2norm(k)
        beta = torch.sigmoid(torch.randn(B, H, L, **f32))
        if gated is None or gated:
            g = torch.rand(B, H, L, **f32) * (-g_low) + g_low
    elif mode == "la":
        s = 1.0 / math.sqrt(dk)
        q, k, v = q * s, k * s, v * s
        if gated:
            g = torch.rand(B, H, L, **f32) * (-g_low) + g_low
    else:
        raise ValueError(mode)
    st = torch.randn(B, H, dk, dv, **f32) * 0.1 if s0 else None
    return dict(q=q.to(in_dtype).contiguous(), k=k.to(in_dtype).contiguous(),
                v=v.to(in_dtype).contiguous(), beta=beta, g=g, s0=st)


# Packed variable-length Gated DeltaNet prefill: 24 sequences (log-uniform length mix
# over two decades, each at least 64 tokens) summing to 32768 tokens per head, 16 heads,
# dk = dv = 128, C = 64.
VARLEN_WORKLOAD = dict(name="gdn_varlen_bf16_N24_H16_T32768_d128", N=24, H=16, T=32768, min_len=64,
                       seed=SEED_BASE + 5)


def draw_seqlens(N: int, total: int, *, seed: int = SEED_BASE, min_len: int = 1) -> list:
    """N sequence lengths >= min_len summing to ``total``, with a long-tailed mix
    (log-uniform weights over two decades), drawn from a seeded CPU generator."""
    if N * min_len > total:
        raise ValueError("total is too small for N sequences of min_len")
    gen = torch.Generator("cpu").manual_seed(int(seed))
    w = torch.exp(torch.rand(N, generator=gen, dtype=torch.float64) * math.log(100.0))
    extra = total - N * min_len
    lens = [min_len + int(x) for x in torch.floor(w / w.sum() * extra).tolist()]
    lens[int(torch.argmax(w))] += total - sum(lens)
    return lens


def make_varlen_inputs(lens, H: int, dk: int, dv: int, *, mode: str = "gdn",
                       in_dtype: torch.dtype = torch.bfloat16, s0: bool = False, seed: int = SEED_BASE,
                       device="cpu", gated: Optional[bool] = None, g_low: float = -0.05,
                       pad: int = 0) -> dict:
    """Draw one packed variable-length batch with the distributions of
    :func:`make_prefill_inputs`: head-major (H, T, d) tensors with T = sum(lens) + pad
    (``pad`` trailing rows belong to no sequence), cu_seqlens (N + 1,) int32 and
    s0 (N, H, dk, dv) when asked."""
    T = int(sum(lens)) + int(pad)
    d = make_prefill_inputs(1, H, T, dk, dv, mode=mode, in_dtype=in_dtype, s0=False, seed=seed,
                            device=device, gated=gated, g_low=g_low)
    out = {name: (None if x is None else x[0].contiguous()) for name, x in d.items() if name != "s0"}
    cu = [0]
    for n in lens:
        cu.append(cu[-1] + int(n))
    out["cu_seqlens"] = torch.tensor(cu, dtype=torch.int32, device=device)
    out["s0"] = None
    if s0:
        gen = _gen(seed + 7, device)
        out["s0"] = torch.randn(len(lens), H, dk, dv, dtype=torch.float32, device=device, generator=gen) * 0.1
    return out


def make_gate_per_key(lead: tuple, L: int, dk: int, *, seed: int = SEED_BASE, g_low: float = -0.05,
                      device="cpu") -> torch.Tensor:
    """Vector-valued log-decays g (*lead, L, dk) fp32 ~ U(g_low, 0), one per token and key
    coordinate (the scalar gate's distribution, drawn per coordinate)."""
    gen = _gen(seed, device)
    return g_low * torch.rand(*lead, L, dk, dtype=torch.float32, device=device, generator=gen)


def make_dskip(H: int, dv: int, *, seed: int = SEED_BASE, device="cpu") -> torch.Tensor:
    """Skip-term weights D (H, dv) fp32 ~ N(0, 1) for the output option o_t += D_h v_t (the
    pages give no distribution for them)."""
    return torch.randn(H, dv, dtype=torch.float32, device=device, generator=_gen(seed, device))


def make_decode_inputs(N: int, H: int, dk: int, dv: int, steps: int, *,
                       in_dtype: torch.dtype = torch.bfloat16, seed: int = SEED_BASE + 4,
                       device="cpu", delta: bool = True, gated: bool = True) -> dict:
    """Draw ``steps`` single-token decode inputs for N sequences plus an initial state.

    q, k: (steps, N, H, dk) unit-norm; v: (steps, N, H, dv) ~ N(0,1);
    beta, g: (steps, N, H) fp32; state: (N, H, dk, dv) fp32 ~ N(0, 0.01).
    """
    gen = _gen(seed, device)
    f32 = dict(dtype=torch.float32, device=device, generator=gen)
    state = torch.randn(N, H, dk, dv, **f32) * 0.1
    q = _l2norm(torch.randn(steps, N, H, dk, **f32)).to(in_dtype)
    k = _l2norm(torch.randn(steps, N, H, dk, **f32)).to(in_dtype)
    v = torch.randn(steps, N, H, dv, **f32).to(in_dtype)
    beta = torch.sigmoid(torch.randn(steps, N, H, **f32)) if delta else None
    g = (torch.rand(steps, N, H, **f32) * 0.05 - 0.05) if gated else None
    return dict(q=q.contiguous(), k=k.contiguous(), v=v.contiguous(), beta=beta, g=g,
                state=state.contiguous())


def make_workload_inputs(w: Workload, device="cpu", steps: Optional[int] = None) -> dict:
    """Inputs of a standard workload, seeded with 1000 + its index."""
    seed = SEED_BASE + w.index
    if w.mode == "decode":
        return make_decode_inputs(w.B, w.H, w.dk, w.dv, steps or w.L, in_dtype=w.in_dtype,
                                  seed=seed, device=device)
    return make_prefill_inputs(w.B, w.H, w.L, w.dk, w.dv, mode=w.mode, in_dtype=w.in_dtype,
                               s0=w.s0, seed=seed, device=device)
