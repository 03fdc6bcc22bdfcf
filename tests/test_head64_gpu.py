"""GPU parity of bf16 calls with head sizes of 64 (dk or dv = 64, chunk 64) against the fp64
oracle, through the C ABI. Such calls run on the tensor-core kernels through copies of the
operands zero-padded to 128: zero key coordinates and zero value columns change no product the
first dk x dv entries depend on, so the padded call's output and final state, cropped, are the
results of the call. Gated DeltaNet with the plain fp32 output and a scalar gate, on batches of
enough (sequence, head) pairs for the one-CTA kernel, skips the copies: that kernel reads the
64-wide tiles directly and stores only dk x dv states and dv output columns, and must give the
padded call's bits. Cases: Gated DeltaNet and linear attention at 64 x 64, 64 x 128 and
128 x 64, with and without S0, ragged and one-token lengths; the packed layout; vector-valued
gates; bf16 output with the skip term; S_final written in place over S0; the output
normalisation (which runs on the fp32 chunk kernel); the direct form against the oracle and
against the padded form, packed, and at the benchmark's size. Bound 2e-3 (bf16 output: + 2^-8)."""
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


# ---- the direct (copy-free) form: Gated DeltaNet, fp32 output, at least 50 (sequence, head) pairs


@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64)])
@pytest.mark.parametrize("L,with_s0,gated", [(130, True, True), (1, True, True), (257, False, False)])
def test_direct_head_sizes(lib, dk, dv, L, with_s0, gated):
    B, H = 4, 16
    inp = W.make_prefill_inputs(B, H, L, dk, dv, mode="gdn", in_dtype=torch.bfloat16, s0=with_s0,
                                seed=860 + L + dk + dv)
    g = inp["g"] if gated else None
    q, k, v, beta = (inp[n].cuda() for n in ("q", "k", "v", "beta"))
    s0 = inp["s0"].cuda() if with_s0 else None
    sf = torch.full((B, H, dk, dv), float("nan"), device="cuda")
    o, sf = lib.gdn_chunk_fwd(q, k, v, beta, None if g is None else g.cuda(), s0=s0, s_final=sf, scale=0.9)
    # the padded form of the same call (a zero skip term adds nothing but takes the copies)
    zero = torch.zeros(H, dv, device="cuda")
    sfp = torch.full((B, H, dk, dv), float("nan"), device="cuda")
    op, sfp = lib.gdn_chunk_fwd(q, k, v, beta, None if g is None else g.cuda(), s0=s0, s_final=sfp, scale=0.9,
                                d_skip=zero)
    assert lib.gdn_sync_status() == 0
    assert torch.equal(o, op) and torch.equal(sf, sfp), "direct and padded forms differ"
    o_ref, s_ref = oracle.recurrent_fwd(inp["q"], inp["k"], inp["v"], inp["beta"], g, inp["s0"], scale=0.9)
    assert _err(o.cpu(), o_ref) <= TOL and _err(sf.cpu(), s_ref) <= TOL


def test_direct_packed_batch(lib):
    lens = [0, 1, 64, 65, 130, 300, 7, 191]
    H = 8
    inp = W.make_varlen_inputs(lens, H, 64, 64, mode="gdn", in_dtype=torch.bfloat16, s0=True, seed=870)
    dev = {n: inp[n].cuda() for n in ("q", "k", "v", "beta", "g", "s0", "cu_seqlens")}
    sf = torch.full((len(lens), H, 64, 64), float("nan"), device="cuda")
    o, sf = lib.gdn_chunk_fwd_varlen(dev["q"], dev["k"], dev["v"], dev["beta"], dev["cu_seqlens"], dev["g"],
                                     s0=dev["s0"], s_final=sf)
    assert lib.gdn_sync_status() == 0
    o_ref, s_ref = oracle.recurrent_fwd_varlen(inp["q"], inp["k"], inp["v"], inp["cu_seqlens"], beta=inp["beta"],
                                               g=inp["g"], s0=inp["s0"])
    assert _err(o.cpu(), o_ref) <= TOL and _err(sf.cpu(), s_ref) <= TOL


def test_direct_full_size_sampled_heads(lib):
    # the benchmark's head-size-64 row: 8 x 16 heads x 4096 tokens, compared on four heads
    B, H, L = 8, 16, 4096
    inp = W.make_prefill_inputs(B, H, L, 64, 64, mode="gdn", in_dtype=torch.bfloat16, seed=W.SEED_BASE + 8)
    dev = {n: inp[n].cuda() for n in ("q", "k", "v", "beta", "g")}
    o = torch.empty(B, H, L, 64, device="cuda")
    sf = torch.empty(B, H, 64, 64, device="cuda")
    lib.gdn_chunk_fwd(dev["q"], dev["k"], dev["v"], dev["beta"], dev["g"], o=o, s_final=sf)
    assert lib.gdn_sync_status() == 0
    o, sf = o.cpu(), sf.cpu()
    for b, h in [(0, 0), (2, 9), (5, 3), (7, 15)]:
        sl = lambda x: x[b:b + 1, h:h + 1]
        o_ref, s_ref = oracle.recurrent_fwd(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["beta"]), sl(inp["g"]))
        assert _err(sl(o), o_ref) <= TOL, f"o head ({b},{h})"
        assert _err(sl(sf), s_ref) <= TOL, f"S head ({b},{h})"


def test_direct_in_place_state(lib):
    # S_final written over S0 (the same buffer) on the direct form: the kernel reads S0 before
    # any chunk and writes S_final after the last
    B, H, L = 4, 16, 100
    inp = W.make_prefill_inputs(B, H, L, 64, 128, mode="gdn", in_dtype=torch.bfloat16, s0=True, seed=880)
    q, k, v, beta, g = (inp[n].cuda() for n in ("q", "k", "v", "beta", "g"))
    state = inp["s0"].cuda().clone()
    o, sf = lib.gdn_chunk_fwd(q, k, v, beta, g, s0=state, s_final=state)
    assert lib.gdn_sync_status() == 0
    o_ref, s_ref = oracle.recurrent_fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["g"], inp["s0"])
    assert _err(o.cpu(), o_ref) <= TOL and _err(state.cpu(), s_ref) <= TOL


@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64)])
@pytest.mark.parametrize("gated", [True, False])
def test_direct_linear_attention_matches_padded(lib, dk, dv, gated):
    # linear attention with the plain fp32 output reads the 64-wide tiles directly on any batch;
    # a zero skip term takes the padded copies: both must give the same bits
    B, H, L = 2, 3, 200
    inp = W.make_prefill_inputs(B, H, L, dk, dv, mode="la", in_dtype=torch.bfloat16, s0=True, seed=890 + dk + dv,
                                gated=gated)
    q, k, v, s0 = (inp[n].cuda() for n in ("q", "k", "v", "s0"))
    g = inp["g"].cuda() if gated else None
    o, sf = lib.lin_attn_chunk_fwd(q, k, v, g, s0=s0, s_final=torch.empty(B, H, dk, dv, device="cuda"))
    op, sfp = lib.lin_attn_chunk_fwd(q, k, v, g, s0=s0, s_final=torch.empty(B, H, dk, dv, device="cuda"),
                                     d_skip=torch.zeros(H, dv, device="cuda"))
    assert lib.gdn_sync_status() == 0
    assert torch.equal(o, op) and torch.equal(sf, sfp), "direct and padded forms differ"
    o_ref, s_ref = oracle.recurrent_fwd(inp["q"], inp["k"], inp["v"], None, inp["g"] if gated else None, inp["s0"])
    assert _err(o.cpu(), o_ref) <= TOL and _err(sf.cpu(), s_ref) <= TOL
