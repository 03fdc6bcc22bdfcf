"""GPU parity of vector-valued gates (one log-decay per key coordinate; row j of the state
decays by exp(g_t[j])), through the C ABI, against the fp64 oracle. These calls run on the
fp32 chunk kernel for every input dtype and size: bf16 inputs with dk = dv = 128 and C = 64,
fp32 inputs at other head sizes and chunk lengths, dense and packed layouts, strong decay,
and together with the output options. Bounds as in test_parity_gpu.py (2e-3 for bf16
inputs, 1e-5 for fp32 inputs; the bf16 output adds 2^-8)."""
import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_sequence_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL = {torch.bfloat16: 2e-3, torch.float32: 1e-5}


@pytest.fixture(scope="module")
def lib():
    from gated_deltanet_sequence_b200 import _lib
    return _lib


def _run(lib, inp, g, chunk, **kw):
    q, k, v, beta, s0 = (None if inp[n] is None else inp[n].cuda() for n in ("q", "k", "v", "beta", "s0"))
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    sf = torch.full((B, H, dk, dv), float("nan"), device="cuda")
    o = torch.full((B, H, L, dv), float("nan"), device="cuda", dtype=kw.pop("odt", torch.float32))
    if beta is not None:
        lib.gdn_chunk_fwd(q, k, v, beta, g.cuda(), o=o, s0=s0, s_final=sf, chunk=chunk, **kw)
    else:
        lib.lin_attn_chunk_fwd(q, k, v, g.cuda(), o=o, s0=s0, s_final=sf, chunk=chunk, **kw)
    assert lib.gdn_sync_status() == 0
    return o.cpu(), sf.cpu()


def _err(x, ref):
    return oracle.max_norm_err(x.float().numpy(), ref)


@pytest.mark.parametrize("delta", [True, False])
@pytest.mark.parametrize("dk,dv,chunk,L,dtype", [
    (128, 128, 64, 130, torch.bfloat16), (64, 64, 64, 200, torch.float32),
    (128, 64, 32, 97, torch.float32), (64, 128, 7, 50, torch.float32), (64, 64, 1, 20, torch.float32),
])
def test_vector_gate_against_oracle(lib, delta, dk, dv, chunk, L, dtype):
    inp = W.make_prefill_inputs(2, 3, L, dk, dv, mode="gdn", in_dtype=dtype, s0=True, seed=80 + L)
    if not delta:
        inp["beta"] = None
    g = W.make_gate_per_key((2, 3), L, dk, seed=81 + L, g_low=-0.2)
    o, sf = _run(lib, inp, g, chunk)
    o_ref, s_ref = oracle.recurrent_fwd(inp["q"], inp["k"], inp["v"], inp["beta"], g, inp["s0"])
    assert _err(o, o_ref) <= TOL[dtype], f"o: {_err(o, o_ref):.3e}"
    assert _err(sf, s_ref) <= TOL[dtype], f"S: {_err(sf, s_ref):.3e}"


@pytest.mark.parametrize("delta", [True, False])
def test_strong_per_coordinate_decay_stays_finite(lib, delta):
    # log-decays down to -8 per token: cumulative decays far below fp32's range inside a chunk
    inp = W.make_prefill_inputs(1, 2, 150, 64, 64, mode="gdn", in_dtype=torch.float32, s0=True, seed=90)
    if not delta:
        inp["beta"] = None
    g = W.make_gate_per_key((1, 2), 150, 64, seed=91, g_low=-8.0)
    o, sf = _run(lib, inp, g, 64)
    assert torch.isfinite(o).all() and torch.isfinite(sf).all()
    o_ref, s_ref = oracle.recurrent_fwd(inp["q"], inp["k"], inp["v"], inp["beta"], g, inp["s0"])
    assert _err(o, o_ref) <= 1e-5 and _err(sf, s_ref) <= 1e-5


def test_equal_coordinates_match_the_scalar_gate(lib):
    # fp32 inputs: the scalar-gate and vector-gate forms of the fp32 kernel agree closely
    inp = W.make_prefill_inputs(2, 2, 130, 64, 64, mode="gdn", in_dtype=torch.float32, s0=True, seed=92)
    g = inp["g"]
    o_s, s_s = _run(lib, inp, g, 64)
    o_v, s_v = _run(lib, inp, g[..., None].expand(*g.shape, 64).contiguous(), 64)
    assert _err(o_v, o_s.double().numpy()) <= 1e-6 and _err(s_v, s_s.double().numpy()) <= 1e-6


def test_vector_gate_with_output_options(lib):
    inp = W.make_prefill_inputs(1, 3, 100, 128, 128, mode="gdn", in_dtype=torch.bfloat16, s0=True, seed=93)
    g = W.make_gate_per_key((1, 3), 100, 128, seed=94)
    D = W.make_dskip(3, 128, seed=95)
    o32, sf32 = _run(lib, inp, g, 64, d_skip=D.cuda())
    ob, sfb = _run(lib, inp, g, 64, d_skip=D.cuda(), odt=torch.bfloat16)
    o_ref, s_ref = oracle.recurrent_fwd(inp["q"], inp["k"], inp["v"], inp["beta"], g, inp["s0"], d_skip=D)
    assert _err(o32, o_ref) <= 2e-3 and _err(sf32, s_ref) <= 2e-3
    assert torch.equal(ob, o32.to(torch.bfloat16)) and torch.equal(sfb, sf32)


@pytest.mark.parametrize("delta", [True, False])
def test_vector_gate_packed_batch(lib, delta):
    lens, pad = [1, 63, 64, 65, 0, 130, 7], 5
    inp = W.make_varlen_inputs(lens, 2, 64, 64, mode="gdn", in_dtype=torch.float32, s0=True, seed=96, pad=pad)
    H, T, dk = inp["q"].shape
    g = W.make_gate_per_key((H,), T, dk, seed=97, g_low=-0.3)
    beta = inp["beta"] if delta else None
    o_ref, s_ref = oracle.recurrent_fwd_varlen(inp["q"], inp["k"], inp["v"], inp["cu_seqlens"], beta, g, inp["s0"])
    dev = {n: inp[n].cuda() for n in ("q", "k", "v", "s0", "cu_seqlens")}
    o = torch.full((H, T, dk), 7.0, device="cuda")
    sf = torch.full(tuple(inp["s0"].shape), float("nan"), device="cuda")
    if delta:
        lib.gdn_chunk_fwd_varlen(dev["q"], dev["k"], dev["v"], beta.cuda(), dev["cu_seqlens"], g.cuda(), o=o,
                                 s0=dev["s0"], s_final=sf)
    else:
        lib.lin_attn_chunk_fwd_varlen(dev["q"], dev["k"], dev["v"], dev["cu_seqlens"], g.cuda(), o=o, s0=dev["s0"],
                                      s_final=sf)
    assert lib.gdn_sync_status() == 0
    used = int(sum(lens))
    o = o.cpu()
    assert torch.all(o[:, used:] == 7.0)
    assert oracle.max_norm_err(o[:, :used].numpy(), o_ref[:, :used]) <= 1e-5
    assert oracle.max_norm_err(sf.cpu().numpy(), s_ref) <= 1e-5


# ---------------------------------------------------------------- decode step options
@pytest.mark.parametrize("delta", [True, False])
@pytest.mark.parametrize("dk,dv,dtype", [(128, 128, torch.bfloat16), (64, 128, torch.float32)])
def test_decode_vector_gate(lib, delta, dk, dv, dtype):
    inp = W.make_decode_inputs(3, 5, dk, dv, 6, in_dtype=dtype, seed=98, device="cuda", delta=delta)
    gv = W.make_gate_per_key((6, 3, 5), 1, dk, seed=99, g_low=-0.3)[..., 0, :].contiguous().cuda()
    state = inp["state"].clone()
    ref_state = inp["state"].cpu().double().numpy().copy()
    for t in range(6):
        b = inp["beta"][t] if delta else None
        o = lib.gdn_decode_step(inp["q"][t], inp["k"][t], inp["v"][t], b, gv[t], state, scale=0.9)
        assert lib.gdn_sync_status() == 0
        o_ref = oracle.decode_step(inp["q"][t].cpu(), inp["k"][t].cpu(), inp["v"][t].cpu(),
                                   None if b is None else b.cpu(), gv[t].cpu(), ref_state, scale=0.9)
        assert _err(o.cpu(), o_ref) <= TOL[dtype], f"o t={t}: {_err(o.cpu(), o_ref):.3e}"
    assert _err(state.cpu(), ref_state) <= TOL[dtype]


def test_decode_skip_term_and_bf16_output(lib):
    inp = W.make_decode_inputs(4, 3, 128, 128, 3, in_dtype=torch.bfloat16, seed=100, device="cuda")
    D = W.make_dskip(3, 128, seed=101).cuda()
    s32, sb = inp["state"].clone(), inp["state"].clone()
    ref_state = inp["state"].cpu().double().numpy().copy()
    for t in range(3):
        args = (inp["q"][t], inp["k"][t], inp["v"][t], inp["beta"][t], inp["g"][t])
        o32 = lib.gdn_decode_step(*args, s32, d_skip=D)
        ob = lib.gdn_decode_step(*args, sb, d_skip=D, out_dtype=torch.bfloat16)
        assert lib.gdn_sync_status() == 0
        o_ref = oracle.decode_step(*(a.cpu() for a in args), ref_state, d_skip=D.cpu())
        assert _err(o32.cpu(), o_ref) <= 2e-3
        assert ob.dtype == torch.bfloat16 and torch.equal(ob, o32.to(torch.bfloat16))
        assert torch.equal(sb, s32)
    assert _err(s32.cpu(), ref_state) <= 2e-3


def test_decode_equal_coordinates_match_scalar_gate(lib):
    inp = W.make_decode_inputs(2, 4, 64, 64, 3, in_dtype=torch.float32, seed=102, device="cuda")
    sa, sv = inp["state"].clone(), inp["state"].clone()
    for t in range(3):
        args = (inp["q"][t], inp["k"][t], inp["v"][t], inp["beta"][t])
        oa = lib.gdn_decode_step(*args, inp["g"][t], sa)
        ov = lib.gdn_decode_step(*args, inp["g"][t][..., None].expand(2, 4, 64).contiguous(), sv)
        assert _err(ov.cpu(), oa.cpu().double().numpy()) <= 1e-6
    assert _err(sv.cpu(), sa.cpu().double().numpy()) <= 1e-6
