"""GPU parity of bf16 calls with head sizes of 64 (dk or dv = 64, chunk 64) against the fp64
oracle, through the C ABI. Such calls run on the tensor-core kernels through copies of the
operands zero-padded to 128: zero key coordinates and zero value columns change no product the
first dk x dv entries depend on, so the padded call's output and final state, cropped, are the
results of the call. Cases: Gated DeltaNet and linear attention at 64 x 64, 64 x 128 and
128 x 64, with and without S0, ragged and one-token lengths; the packed layout; vector-valued
gates; bf16 output with the skip term; S_final written in place over S0; the output
normalisation (which runs on the fp32 chunk kernel). Bound 2e-3 (bf16 output: + 2^-8)."""
import pytest
import torch

import oracle
from gated_deltanet_sequence_b200 import workloads as W

pytestmark = pytest.mark.gpu
TOL = 2e-3


@pytest.fixture(scope="module")
def lib():
    from gated_deltanet_sequence_b200 import _lib
    return _lib


def _err(x, ref):
    return oracle.max_norm_err(x.float().numpy(), ref)


@pytest.mark.parametrize("mode", ["gdn", "la"])
@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64)])
@pytest.mark.parametrize("L,with_s0", [(1, True), (130, True), (200, False)])
def test_padded_head_sizes(lib, mode, dk, dv, L, with_s0):
    inp = W.make_prefill_inputs(2, 3, L, dk, dv, mode=mode, in_dtype=torch.bfloat16, s0=with_s0, seed=800 + L + dk,
                                gated=True)
    q, k, v, g = (inp[n].cuda() for n in ("q", "k", "v", "g"))
    s0 = inp["s0"].cuda() if with_s0 else None
    sf = torch.full((2, 3, dk, dv), float("nan"), device="cuda")
    if mode == "gdn":
        o, sf = lib.gdn_chunk_fwd(q, k, v, inp["beta"].cuda(), g, s0=s0, s_final=sf, scale=0.8)
    else:
        o, sf = lib.lin_attn_chunk_fwd(q, k, v, g, s0=s0, s_final=sf, scale=0.8)
    assert lib.gdn_sync_status() == 0
    o_ref, s_ref = oracle.recurrent_fwd(inp["q"], inp["k"], inp["v"], inp["beta"] if mode == "gdn" else None,
                                        inp["g"], inp["s0"], scale=0.8)
    assert _err(o.cpu(), o_ref) <= TOL and _err(sf.cpu(), s_ref) <= TOL


@pytest.mark.parametrize("delta", [True, False])
def test_padded_packed_batch(lib, delta):
    lens, pad = [1, 63, 64, 65, 0, 130, 7], 5
    inp = W.make_varlen_inputs(lens, 2, 64, 64, mode="gdn", in_dtype=torch.bfloat16, s0=True, seed=810, pad=pad)
    H, T, dk = inp["q"].shape
    beta = inp["beta"] if delta else None
    o_ref, s_ref = oracle.recurrent_fwd_varlen(inp["q"], inp["k"], inp["v"], inp["cu_seqlens"], beta, inp["g"],
                                               inp["s0"])
    dev = {n: inp[n].cuda() for n in ("q", "k", "v", "g", "s0", "cu_seqlens")}
    o = torch.full((H, T, 64), 7.0, device="cuda")
    sf = torch.full(tuple(inp["s0"].shape), float("nan"), device="cuda")
    if delta:
        lib.gdn_chunk_fwd_varlen(dev["q"], dev["k"], dev["v"], beta.cuda(), dev["cu_seqlens"], dev["g"], o=o,
                                 s0=dev["s0"], s_final=sf)
    else:
        lib.lin_attn_chunk_fwd_varlen(dev["q"], dev["k"], dev["v"], dev["cu_seqlens"], dev["g"], o=o, s0=dev["s0"],
                                      s_final=sf)
    assert lib.gdn_sync_status() == 0
    used = int(sum(lens))
    assert oracle.max_norm_err(o[:, :used].cpu().numpy(), o_ref[:, :used]) <= TOL
    assert oracle.max_norm_err(sf.cpu().numpy(), s_ref) <= TOL


def test_padded_vector_gates(lib):
    inp = W.make_prefill_inputs(1, 3, 150, 64, 64, mode="gdn", in_dtype=torch.bfloat16, s0=True, seed=820)
    g = W.make_gate_per_key((1, 3), 150, 64, seed=821, g_low=-0.2)
    q, k, v, beta, s0 = (inp[n].cuda() for n in ("q", "k", "v", "beta", "s0"))
    o, sf = lib.gdn_chunk_fwd(q, k, v, beta, g.cuda(), s0=s0, s_final=torch.empty(1, 3, 64, 64, device="cuda"))
    assert lib.gdn_sync_status() == 0
    o_ref, s_ref = oracle.recurrent_fwd(inp["q"], inp["k"], inp["v"], inp["beta"], g, inp["s0"])
    assert _err(o.cpu(), o_ref) <= TOL and _err(sf.cpu(), s_ref) <= TOL


def test_padded_bf16_output_and_skip_term_in_place_state(lib):
    inp = W.make_prefill_inputs(1, 3, 100, 128, 64, mode="gdn", in_dtype=torch.bfloat16, s0=True, seed=830)
    D = W.make_dskip(3, 64, seed=831)
    q, k, v, beta, g = (inp[n].cuda() for n in ("q", "k", "v", "beta", "g"))
    state = inp["s0"].cuda().clone()
    o32, _ = lib.gdn_chunk_fwd(q, k, v, beta, g, s0=state.clone(), s_final=None, d_skip=D.cuda())
    ob, sf = lib.gdn_chunk_fwd(q, k, v, beta, g, s0=state, s_final=state, d_skip=D.cuda(), out_dtype=torch.bfloat16)
    assert lib.gdn_sync_status() == 0
    o_ref, s_ref = oracle.recurrent_fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["g"], inp["s0"], d_skip=D)
    assert _err(o32.cpu(), o_ref) <= TOL and _err(state.cpu(), s_ref) <= TOL
    assert torch.equal(ob, o32.to(torch.bfloat16))


def test_output_normalisation_at_dv64(lib):
    inp = W.make_prefill_inputs(1, 2, 120, 64, 64, mode="gdn", in_dtype=torch.bfloat16, s0=True, seed=840)
    q, k, v, beta, g, s0 = (inp[n].cuda() for n in ("q", "k", "v", "beta", "g", "s0"))
    o, _ = lib.gdn_chunk_fwd(q, k, v, beta, g, s0=s0, xnorm="rms")
    assert lib.gdn_sync_status() == 0
    o_plain, _ = oracle.recurrent_fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["g"], inp["s0"])
    assert _err(o.cpu(), oracle.xnorm(o_plain, "rms")) <= TOL
