"""GPU parity of the output normalisation (page "LinearAttention 概述", section "The Devil
in Linear Transformer": the normaliser's denominator is dropped and the output is
normalised instead, O = XNorm(Q (K^T V)); reading: each output row of each head
normalised over its dv values, RMS or layer form, times a weight (H, dv), after the skip
term and before the output rounding) on every path: the tensor-core linear-attention
kernel, the one-CTA and cluster forms of the Gated DeltaNet kernel, the fp32 chunk kernel
(whose value slices form a thread-block cluster for the row statistics), packed batches
and the decode step.

Reference: the fp64 oracle's recurrence, skip term and xnorm. Bounds (max-normalised
error): 2e-3 for bf16 inputs, 1e-5 for fp32 inputs; a bf16 output adds 2^-8 (its
rounding), and must equal the fp32 output rounded to bf16 bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_sequence_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL = {torch.bfloat16: 2e-3, torch.float32: 1e-5}
MODES = {"plain": (False, False), "gated": (False, True), "delta": (True, False), "gdn": (True, True)}
# (B, H, L, dk, dv, dtype, chunk): 6 heads -> cluster form of the GDN kernel; 64 heads -> one
# CTA each; fp32 inputs and bf16 inputs at chunk 32 -> the fp32 chunk kernel (2 and 4 slices)
PATHS = {
    "tc_small_heads": (2, 3, 300, 128, 128, torch.bfloat16, 64),
    "tc_many_heads": (1, 64, 130, 128, 128, torch.bfloat16, 64),
    "fp32_kernel_d64": (2, 2, 150, 64, 64, torch.float32, 64),
    "fp32_kernel_d128": (1, 3, 100, 128, 128, torch.bfloat16, 32),
}
EPS = 1e-5


@pytest.fixture(scope="module")
def lib():
    from gated_deltanet_sequence_b200 import _lib
    return _lib


def _inputs(B, H, L, dk, dv, mode, dtype, seed):
    delta, gated = MODES[mode]
    inp = W.make_prefill_inputs(B, H, L, dk, dv, mode="gdn", in_dtype=dtype, s0=True, seed=seed)
    if not delta:
        inp["beta"] = None
    if not gated:
        inp["g"] = None
    return inp


def _run(lib, inp, chunk, out_dtype, **opts):
    q, k, v, beta, g, s0 = (None if inp[n] is None else inp[n].cuda() for n in ("q", "k", "v", "beta", "g", "s0"))
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    o = torch.full((B, H, L, dv), float("nan"), device="cuda", dtype=out_dtype)
    sf = torch.full((B, H, dk, dv), float("nan"), device="cuda")
    if beta is not None:
        lib.gdn_chunk_fwd(q, k, v, beta, g, o=o, s0=s0, s_final=sf, chunk=chunk, **opts)
    else:
        lib.lin_attn_chunk_fwd(q, k, v, g, o=o, s0=s0, s_final=sf, chunk=chunk, **opts)
    assert lib.gdn_sync_status() == 0
    return o.cpu(), sf.cpu()


def _check(x, ref, tol, what):
    err = oracle.max_norm_err(x, ref)
    assert np.isfinite(err) and err <= tol, f"{what}: max-normalised error {err:.3e} > {tol:.1e}"


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("mode", ["plain", "gdn"])
@pytest.mark.parametrize("kind", ["rms", "layer"])
def test_xnorm_dense(lib, path, mode, kind):
    B, H, L, dk, dv, dtype, chunk = PATHS[path]
    seed = 900 + 10 * list(PATHS).index(path) + 2 * list(MODES).index(mode) + (kind == "layer")
    inp = _inputs(B, H, L, dk, dv, mode, dtype, seed=seed)
    gen = torch.Generator().manual_seed(17)
    w = torch.randn(H, dv, generator=gen)
    D = W.make_dskip(H, dv, seed=18)
    opts = dict(xnorm=kind, xnorm_weight=w.cuda(), xnorm_eps=EPS, d_skip=D.cuda())
    o32, s32 = _run(lib, inp, chunk, torch.float32, **opts)
    ob, sb = _run(lib, inp, chunk, torch.bfloat16, **opts)
    o_ref, s_ref = oracle.recurrent_fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["g"], inp["s0"], d_skip=D)
    x_ref = oracle.xnorm(o_ref, kind, w, EPS)
    _check(o32, x_ref, TOL[dtype], f"{path} {mode} {kind} o")
    _check(s32, s_ref, TOL[dtype], f"{path} {mode} {kind} S")
    _check(ob.float(), x_ref, TOL[dtype] + 2.0 ** -8, f"{path} {mode} {kind} bf16 o")
    assert torch.equal(ob, o32.to(torch.bfloat16)), "bf16 output is not the rounded fp32 output"
    assert torch.equal(sb, s32)


@pytest.mark.parametrize("kind", ["rms", "layer"])
def test_xnorm_without_weight_or_skip(lib, kind):
    inp = _inputs(1, 4, 200, 128, 128, "gdn", torch.bfloat16, seed=931)
    o, _ = _run(lib, inp, 64, torch.float32, xnorm=kind, xnorm_eps=EPS)
    o_ref, _ = oracle.recurrent_fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["g"], inp["s0"])
    _check(o, oracle.xnorm(o_ref, kind, None, EPS), 2e-3, f"{kind} unweighted")


@pytest.mark.parametrize("path", ["tc", "fp32_kernel"])
def test_xnorm_varlen(lib, path):
    lens = [70, 0, 129, 5, 64]
    dtype, chunk = (torch.bfloat16, 64) if path == "tc" else (torch.float32, 64)
    d = 128 if path == "tc" else 64
    H = 3
    inp = W.make_varlen_inputs(lens, H, d, d, mode="gdn", in_dtype=dtype, seed=932)
    dev = {n: (None if x is None else x.cuda()) for n, x in inp.items()}
    w = torch.randn(H, d, generator=torch.Generator().manual_seed(19))
    o = torch.zeros(H, inp["q"].shape[1], d, device="cuda")
    lib.gdn_chunk_fwd_varlen(dev["q"], dev["k"], dev["v"], dev["beta"], dev["cu_seqlens"], dev["g"], o=o, chunk=chunk,
                             xnorm="rms", xnorm_weight=w.cuda(), xnorm_eps=EPS)
    assert lib.gdn_sync_status() == 0
    o_ref, _ = oracle.recurrent_fwd_varlen(inp["q"], inp["k"], inp["v"], inp["cu_seqlens"].cpu(), beta=inp["beta"],
                                           g=inp["g"])
    cu = inp["cu_seqlens"].tolist()
    inside = np.zeros(o_ref.shape[1], bool)
    inside[: cu[-1]] = True
    x_ref = oracle.xnorm(o_ref[:, inside], "rms", w, EPS)
    _check(o.cpu()[:, inside], x_ref, TOL[dtype], f"varlen {path}")


@pytest.mark.parametrize("dk,dv,dtype", [(128, 128, torch.bfloat16), (128, 64, torch.float32)])
@pytest.mark.parametrize("kind", ["rms", "layer"])
def test_xnorm_decode(lib, dk, dv, dtype, kind):
    inp = W.make_decode_inputs(3, 4, dk, dv, 5, in_dtype=dtype, seed=933, device="cuda")
    w = torch.randn(4, dv, generator=torch.Generator().manual_seed(20))
    state = inp["state"].clone()
    ref_state = inp["state"].cpu().double().numpy().copy()
    for t in range(5):
        args = [inp[n][t] for n in ("q", "k", "v", "beta", "g")]
        o = lib.gdn_decode_step(*args, state, xnorm=kind, xnorm_weight=w.cuda(), xnorm_eps=EPS)
        o_ref = oracle.decode_step(*(a.cpu() for a in args), ref_state)
        x_ref = oracle.xnorm(o_ref[:, :, None, :], kind, w, EPS)[:, :, 0, :]   # rows of (N, H, 1, dv)
        _check(o.cpu(), x_ref, TOL[dtype], f"decode {kind} step {t}")
    assert lib.gdn_sync_status() == 0
    _check(state.cpu(), ref_state, TOL[dtype], "decode state")


def test_xnorm_rejects_bad_options(lib):
    inp = _inputs(1, 2, 64, 128, 128, "gdn", torch.bfloat16, seed=934)
    with pytest.raises(Exception):
        _run(lib, inp, 64, torch.float32, xnorm="rms", xnorm_eps=0.0)
    with pytest.raises(ValueError):
        _run(lib, inp, 64, torch.float32, xnorm="l2")
