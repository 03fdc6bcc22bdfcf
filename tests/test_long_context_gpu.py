"""GPU parity of long sequences over few heads against the fp64 oracle, through the C ABI.

Dense bf16 calls at dk = dv = 128, chunk 64, whose heads number at most a third of the SMs and
whose sequences have at least 128 chunks run on the per-chunk prep kernel and the per-head
chain kernel, cut into segments of 64 chunks: the prep of segment i + 1 runs on a second
stream while the chain takes segment i, and the state crosses segments through a workspace
buffer. Cases: Gated DeltaNet with a scalar gate, without a gate, with vector-valued gates, and
gated linear attention; a ragged last segment; an initial state; the output options. Bound
2e-3 (max-norm relative error), as for the other bf16 tensor-core kernels."""
import pytest
import torch

import oracle
from gated_deltanet_sequence_b200 import workloads as W

pytestmark = pytest.mark.gpu
TOL = 2e-3
L_LONG = 2 * 64 * 64 + 70   # three segments: 64, 64 and 2 chunks, the last one ragged


@pytest.fixture(scope="module")
def lib():
    from gated_deltanet_sequence_b200 import _lib
    return _lib


def _err(x, ref):
    return oracle.max_norm_err(x.float().numpy(), ref)


def _run(lib, inp, g, delta, **kw):
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    s0 = None if inp.get("s0") is None else inp["s0"].cuda()
    B, H, L, dk = q.shape
    sf = torch.full((B, H, dk, 128), float("nan"), device="cuda")
    o = torch.full((B, H, L, 128), float("nan"), device="cuda", dtype=kw.pop("odt", torch.float32))
    gg = None if g is None else g.cuda()
    if delta:
        lib.gdn_chunk_fwd(q, k, v, inp["beta"].cuda(), gg, o=o, s0=s0, s_final=sf, **kw)
    else:
        lib.lin_attn_chunk_fwd(q, k, v, gg, o=o, s0=s0, s_final=sf, **kw)
    assert lib.gdn_sync_status() == 0
    return o.cpu(), sf.cpu()


@pytest.mark.parametrize("kind", ["scalar", "ungated", "vector", "la_vector"])
def test_segmented_long_sequence(lib, kind):
    delta = kind != "la_vector"
    inp = W.make_prefill_inputs(1, 3, L_LONG, 128, 128, mode="gdn", in_dtype=torch.bfloat16, s0=True,
                                seed=600 + len(kind))
    if kind == "scalar":
        g = inp["g"]
    elif kind == "ungated":
        g = None
    else:
        g = W.make_gate_per_key((1, 3), L_LONG, 128, seed=601, g_low=-0.1)
    beta = inp["beta"] if delta else None
    o, sf = _run(lib, inp, g, delta, scale=0.9)
    o_ref, s_ref = oracle.recurrent_fwd(inp["q"], inp["k"], inp["v"], beta, g, inp["s0"], scale=0.9)
    eo, es = _err(o, o_ref), _err(sf, s_ref)
    assert eo <= TOL and es <= TOL, f"{kind}: o {eo:.3e}  S {es:.3e}"


def test_segmented_strong_scalar_decay(lib):
    # log-decays of -30 per token: every chunk takes exp(G_r - G_s) per element
    inp = W.make_prefill_inputs(1, 2, L_LONG, 128, 128, mode="gdn", in_dtype=torch.bfloat16, s0=True, seed=610)
    g = torch.full_like(inp["g"], -30.0)
    o, sf = _run(lib, inp, g, True)
    assert torch.isfinite(o).all() and torch.isfinite(sf).all()
    o_ref, s_ref = oracle.recurrent_fwd(inp["q"], inp["k"], inp["v"], inp["beta"], g, inp["s0"])
    assert _err(o, o_ref) <= TOL and _err(sf, s_ref) <= TOL


def test_segmented_output_options(lib):
    inp = W.make_prefill_inputs(1, 2, L_LONG, 128, 128, mode="gdn", in_dtype=torch.bfloat16, s0=True, seed=620)
    D = W.make_dskip(2, 128, seed=621)
    o32, sf32 = _run(lib, inp, inp["g"], True, d_skip=D.cuda())
    ob, sfb = _run(lib, inp, inp["g"], True, d_skip=D.cuda(), odt=torch.bfloat16)
    o_ref, s_ref = oracle.recurrent_fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["g"], inp["s0"], d_skip=D)
    assert _err(o32, o_ref) <= TOL and _err(sf32, s_ref) <= TOL
    assert torch.equal(ob, o32.to(torch.bfloat16)) and torch.equal(sfb, sf32)


def test_segments_agree_with_the_one_cta_kernel(lib):
    # the same three heads inside a 64-head batch take the one-CTA kernel; both forms agree
    # with each other as closely as each agrees with the oracle
    L = 64 * 130
    small = W.make_prefill_inputs(1, 3, L, 128, 128, mode="gdn", in_dtype=torch.bfloat16, s0=True, seed=630)
    big = W.make_prefill_inputs(1, 64, L, 128, 128, mode="gdn", in_dtype=torch.bfloat16, s0=True, seed=631)
    for name in ("q", "k", "v", "beta", "g", "s0"):
        big[name][:, :3] = small[name]
    o1, s1 = _run(lib, small, small["g"], True)
    o2, s2 = _run(lib, big, big["g"], True)
    assert _err(o1, o2[:, :3].double().numpy()) <= TOL and _err(s1, s2[:, :3].double().numpy()) <= TOL


@pytest.mark.parametrize("L,B,H,with_s0", [(128 * 64, 1, 2, True), (128 * 64 + 1, 2, 3, False),
                                           (192 * 64 - 5, 1, 4, True)])
def test_segment_boundaries(lib, L, B, H, with_s0):
    # exactly two segments; one token past them (a one-token third segment) over two sequences;
    # a ragged third segment
    inp = W.make_prefill_inputs(B, H, L, 128, 128, mode="gdn", in_dtype=torch.bfloat16, s0=with_s0,
                                seed=640 + L % 97)
    o, sf = _run(lib, inp, inp["g"], True)
    o_ref, s_ref = oracle.recurrent_fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["g"], inp["s0"])
    eo, es = _err(o, o_ref), _err(sf, s_ref)
    assert eo <= TOL and es <= TOL, f"L={L}: o {eo:.3e}  S {es:.3e}"


def test_segmented_vector_gates_without_initial_state(lib):
    L = 128 * 64 + 33
    inp = W.make_prefill_inputs(1, 2, L, 128, 128, mode="gdn", in_dtype=torch.bfloat16, s0=False, seed=650)
    g = W.make_gate_per_key((1, 2), L, 128, seed=651, g_low=-0.3)
    o, sf = _run(lib, inp, g, True)
    o_ref, s_ref = oracle.recurrent_fwd(inp["q"], inp["k"], inp["v"], inp["beta"], g, None)
    assert _err(o, o_ref) <= TOL and _err(sf, s_ref) <= TOL
