"""GPU parity of the tensor-core form for vector-valued gates (one log-decay per token and key
coordinate) against the fp64 oracle, through the C ABI. Dense bf16 batches with
dk = dv = 128 and chunk 64 take this form: a per-chunk prep kernel (decay-weighted Gram on the
tensor cores with the per-coordinate factors, the coordinates whose decay range in a chunk
exceeds what fp16 factors hold done exactly on the CUDA cores) and a per-head chain kernel.

Cases: ragged lengths (one token, one chunk, a ragged tail), an initial state, Gated DeltaNet
and gated linear attention; chunks whose every coordinate takes the factored Gram, chunks
with a few exactly-handled coordinates, chunks with more of them than the mixed form takes
(the whole Gram then exact), and sequences that mix the three; the output options; and the
benchmark's full size (8 x 16 heads x 4096 tokens) on sampled heads. Bound 2e-3 (max-norm
relative error), as for the scalar-gate tensor-core kernels."""
import numpy as np
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


def _run(lib, inp, g, delta=True, **kw):
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    s0 = None if inp.get("s0") is None else inp["s0"].cuda()
    B, H, L, dk = q.shape
    sf = torch.full((B, H, dk, 128), float("nan"), device="cuda")
    o = torch.full((B, H, L, 128), float("nan"), device="cuda", dtype=kw.pop("odt", torch.float32))
    if delta:
        lib.gdn_chunk_fwd(q, k, v, inp["beta"].cuda(), g.cuda(), o=o, s0=s0, s_final=sf, **kw)
    else:
        lib.lin_attn_chunk_fwd(q, k, v, g.cuda(), o=o, s0=s0, s_final=sf, **kw)
    assert lib.gdn_sync_status() == 0
    return o.cpu(), sf.cpu()


def _err(x, ref):
    return oracle.max_norm_err(x.float().numpy(), ref)


def _check(lib, inp, g, delta=True, **kw):
    o, sf = _run(lib, inp, g, delta, **kw)
    o_ref, s_ref = oracle.recurrent_fwd(inp["q"], inp["k"], inp["v"], inp["beta"] if delta else None, g, inp["s0"],
                                        scale=kw.get("scale", 1.0), d_skip=kw.get("d_skip"))
    eo, es = _err(o, o_ref), _err(sf, s_ref)
    assert eo <= TOL and es <= TOL, f"o {eo:.3e}  S {es:.3e}"
    return eo, es


def _inputs(B, H, L, seed, mode="gdn", s0=True):
    inp = W.make_prefill_inputs(B, H, L, 128, 128, mode=mode, in_dtype=torch.bfloat16, s0=s0, seed=seed,
                                gated=True)
    if mode == "la":
        inp["beta"] = None
    return inp


@pytest.mark.parametrize("delta", [True, False])
@pytest.mark.parametrize("L,g_low", [(1, -0.05), (64, -0.05), (130, -0.05), (257, -0.2)])
def test_factored_gram(lib, delta, L, g_low):
    inp = _inputs(2, 3, L, 300 + L, "gdn" if delta else "la")
    g = W.make_gate_per_key((2, 3), L, 128, seed=301 + L, g_low=g_low)
    _check(lib, inp, g, delta, scale=0.8)


@pytest.mark.parametrize("delta", [True, False])
@pytest.mark.parametrize("n_strong", [1, 9, 32])
def test_some_coordinates_exact(lib, delta, n_strong):
    # n_strong coordinates decay by up to e^-3 per token: their range over a chunk exceeds the
    # factored form's, so their terms are added exactly next to the UMMA Gram
    inp = _inputs(1, 3, 200, 310 + n_strong, "gdn" if delta else "la")
    g = W.make_gate_per_key((1, 3), 200, 128, seed=311 + n_strong)
    idx = torch.randperm(128, generator=torch.Generator().manual_seed(n_strong))[:n_strong]
    g[..., idx] = W.make_gate_per_key((1, 3), 200, n_strong, seed=312, g_low=-3.0)
    _check(lib, inp, g, delta)


@pytest.mark.parametrize("delta", [True, False])
def test_every_coordinate_exact(lib, delta):
    # log-decays down to -8 per token on every coordinate: cumulative decays far below fp32's
    # range inside a chunk; the whole Gram of every chunk is formed exactly
    inp = _inputs(1, 2, 150, 320, "gdn" if delta else "la")
    g = W.make_gate_per_key((1, 2), 150, 128, seed=321, g_low=-8.0)
    o, sf = _run(lib, inp, g, delta)
    assert torch.isfinite(o).all() and torch.isfinite(sf).all()
    _check(lib, inp, g, delta)


def test_chunks_of_each_kind_in_one_sequence(lib):
    # tokens 0-99 mild, 100-199 a few strong coordinates, 200-299 all strong, 300-330 mild:
    # the state crosses chunks of every kind
    L = 331
    inp = _inputs(2, 2, L, 330)
    g = W.make_gate_per_key((2, 2), L, 128, seed=331)
    g[..., 100:200, :40] = W.make_gate_per_key((2, 2), 100, 40, seed=332, g_low=-2.0)
    g[..., 200:300, :] = W.make_gate_per_key((2, 2), 100, 128, seed=333, g_low=-5.0)
    _check(lib, inp, g)


def test_output_options(lib):
    inp = _inputs(1, 3, 150, 340)
    g = W.make_gate_per_key((1, 3), 150, 128, seed=341)
    D = W.make_dskip(3, 128, seed=342)
    o32, sf32 = _run(lib, inp, g, d_skip=D.cuda())
    ob, sfb = _run(lib, inp, g, d_skip=D.cuda(), odt=torch.bfloat16)
    o_ref, s_ref = oracle.recurrent_fwd(inp["q"], inp["k"], inp["v"], inp["beta"], g, inp["s0"], d_skip=D)
    assert _err(o32, o_ref) <= TOL and _err(sf32, s_ref) <= TOL
    assert torch.equal(ob, o32.to(torch.bfloat16)) and torch.equal(sfb, sf32)
    ox, _ = _run(lib, inp, g, xnorm="rms")
    o_plain, _ = oracle.recurrent_fwd(inp["q"], inp["k"], inp["v"], inp["beta"], g, inp["s0"])
    assert _err(ox, oracle.xnorm(o_plain, "rms")) <= TOL


def test_equal_coordinates_agree_with_the_scalar_gate(lib):
    # the same decay on every coordinate is the scalar gate: both tensor-core forms agree
    # with each other as closely as each agrees with the oracle
    inp = _inputs(2, 2, 200, 350)
    g = inp["g"]
    o_s, s_s = _run(lib, inp, g)
    o_v, s_v = _run(lib, inp, g[..., None].expand(*g.shape, 128).contiguous())
    assert _err(o_v, o_s.double().numpy()) <= TOL and _err(s_v, s_s.double().numpy()) <= TOL


def test_full_size_sampled_heads(lib):
    # the benchmark's workload (8 x 16 heads x 4096 tokens, g ~ U(-0.05, 0) per coordinate),
    # compared on four heads
    B, H, L = 8, 16, 4096
    w = W.WORKLOADS[2]
    inp = W.make_prefill_inputs(B, H, L, 128, 128, mode="gdn", in_dtype=torch.bfloat16, seed=W.SEED_BASE + 7)
    g = W.make_gate_per_key((B, H), L, 128, seed=W.SEED_BASE + 7)
    dev = {n: inp[n].cuda() for n in ("q", "k", "v", "beta")}
    o = torch.empty(B, H, L, 128, device="cuda")
    sf = torch.empty(B, H, 128, 128, device="cuda")
    lib.gdn_chunk_fwd(dev["q"], dev["k"], dev["v"], dev["beta"], g.cuda(), o=o, s_final=sf)
    assert lib.gdn_sync_status() == 0
    o, sf = o.cpu(), sf.cpu()
    for b, h in [(0, 0), (3, 7), (5, 2), (7, 15)]:
        sl = lambda x: x[b:b + 1, h:h + 1]
        o_ref, s_ref = oracle.recurrent_fwd(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["beta"]), sl(g))
        assert _err(sl(o), o_ref) <= TOL, f"o head ({b},{h})"
        assert _err(sl(sf), s_ref) <= TOL, f"S head ({b},{h})"
    assert w.L == L and w.B == B and w.H == H
