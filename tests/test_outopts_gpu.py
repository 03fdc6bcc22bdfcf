"""GPU parity of the output options: bf16 output, and Mamba's skip term o_t += D_h v_t
(page "【CS336】lecture4", section "继续改进：Mamba"), on every prefill path (tensor-core
linear attention, the one-CTA and cluster forms of the Gated DeltaNet kernel, the fp32
kernel) in the dense and the packed layout.

Bounds (max-normalised error against the fp64 oracle): with fp32 output the usual 2e-3
(bf16 inputs) and 1e-5 (fp32 inputs). A bf16 output adds the rounding of each element to
8 significant bits, at most 2^-8 |o_i| <= 2^-8 max|o|, so its bound is the input bound
plus 2^-8 (5.9e-3 for bf16 inputs, 3.9e-3 for fp32 inputs). Every kernel
forms the bf16 output by rounding (to nearest, ties to even) the fp32 value it stores in
fp32 mode, so the two modes must agree bit for bit after that rounding.
"""
import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_sequence_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL = {torch.bfloat16: 2e-3, torch.float32: 1e-5}
TOL_BF16_OUT = {dt: t + 2.0 ** -8 for dt, t in TOL.items()}
MODES = {"plain": (False, False), "gated": (False, True), "delta": (True, False), "gdn": (True, True)}
# (B, H, L, d, dtype): 6 heads -> cluster form of the GDN kernel; 64 heads -> one CTA each
PATHS = {
    "tc_small_heads": (2, 3, 300, 128, torch.bfloat16),
    "tc_many_heads": (1, 64, 130, 128, torch.bfloat16),
    "fp32_kernel": (2, 2, 150, 64, torch.float32),
}


@pytest.fixture(scope="module")
def lib():
    from gated_deltanet_sequence_b200 import _lib
    return _lib


def _dense(lib, inp, D, out_dtype):
    q, k, v, beta, g, s0 = (None if inp[n] is None else inp[n].cuda() for n in ("q", "k", "v", "beta", "g", "s0"))
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    o = torch.full((B, H, L, dv), float("nan"), device="cuda", dtype=out_dtype)
    sf = torch.full((B, H, dk, dv), float("nan"), device="cuda")
    Dd = None if D is None else D.cuda()
    if beta is not None:
        lib.gdn_chunk_fwd(q, k, v, beta, g, o=o, s0=s0, s_final=sf, d_skip=Dd)
    else:
        lib.lin_attn_chunk_fwd(q, k, v, g, o=o, s0=s0, s_final=sf, d_skip=Dd)
    assert lib.gdn_sync_status() == 0
    return o.cpu(), sf.cpu()


def _inputs(B, H, L, d, mode, dtype, seed):
    delta, gated = MODES[mode]
    inp = W.make_prefill_inputs(B, H, L, d, d, mode="gdn", in_dtype=dtype, s0=True, seed=seed)
    if not delta:
        inp["beta"] = None
    if not gated:
        inp["g"] = None
    return inp


def _err(x, ref):
    return oracle.max_norm_err(x.float().numpy() if torch.is_tensor(x) else x, ref)


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("mode", ["gdn", "delta", "gated", "plain"])
def test_skip_term_and_bf16_output(lib, path, mode):
    B, H, L, d, dt = PATHS[path]
    inp = _inputs(B, H, L, d, mode, dt, seed=70 + L)
    D = W.make_dskip(H, d, seed=71)
    o_ref, s_ref = oracle.recurrent_fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["g"], inp["s0"],
                                        d_skip=D)
    o32, sf32 = _dense(lib, inp, D, torch.float32)
    assert _err(o32, o_ref) <= TOL[dt], f"o (skip, fp32 out): {_err(o32, o_ref):.3e}"
    assert _err(sf32, s_ref) <= TOL[dt], f"S (skip, fp32 out): {_err(sf32, s_ref):.3e}"
    ob, sfb = _dense(lib, inp, D, torch.bfloat16)
    assert torch.equal(ob, o32.to(torch.bfloat16)), "bf16 output is not the rounded fp32 output"
    assert torch.equal(sfb, sf32), "the output option changed the final state"
    assert _err(ob, o_ref) <= TOL_BF16_OUT[dt]
    # bf16 output without the skip term, against the plain oracle
    o_ref0, _ = oracle.recurrent_fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["g"], inp["s0"])
    o32n, _ = _dense(lib, inp, None, torch.float32)
    obn, _ = _dense(lib, inp, None, torch.bfloat16)
    assert torch.equal(obn, o32n.to(torch.bfloat16))
    assert _err(obn, o_ref0) <= TOL_BF16_OUT[dt]


@pytest.mark.parametrize("mode", ["gdn", "plain"])
@pytest.mark.parametrize("d,dt", [(128, torch.bfloat16), (64, torch.float32)])
def test_packed_batch_output_options(lib, mode, d, dt):
    lens, pad = [1, 63, 64, 65, 0, 130, 7], 5
    delta, gated = MODES[mode]
    inp = W.make_varlen_inputs(lens, 3, d, d, mode="gdn", in_dtype=dt, s0=True, seed=75, pad=pad)
    if not delta:
        inp["beta"] = None
    if not gated:
        inp["g"] = None
    D = W.make_dskip(3, d, seed=76)
    o_ref, s_ref = oracle.recurrent_fwd_varlen(inp["q"], inp["k"], inp["v"], inp["cu_seqlens"], inp["beta"],
                                               inp["g"], inp["s0"], d_skip=D)
    dev = {n: (None if inp[n] is None else inp[n].cuda()) for n in ("q", "k", "v", "beta", "g", "s0", "cu_seqlens")}
    H, T, _ = inp["q"].shape
    outs = {}
    for odt in (torch.float32, torch.bfloat16):
        o = torch.full((H, T, d), 7.0, device="cuda", dtype=odt)     # sentinel: rows of no sequence
        sf = torch.full(tuple(inp["s0"].shape), float("nan"), device="cuda")
        if delta:
            lib.gdn_chunk_fwd_varlen(dev["q"], dev["k"], dev["v"], dev["beta"], dev["cu_seqlens"], dev["g"], o=o,
                                     s0=dev["s0"], s_final=sf, d_skip=D.cuda())
        else:
            lib.lin_attn_chunk_fwd_varlen(dev["q"], dev["k"], dev["v"], dev["cu_seqlens"], dev["g"], o=o,
                                          s0=dev["s0"], s_final=sf, d_skip=D.cuda())
        assert lib.gdn_sync_status() == 0
        outs[odt] = (o.cpu(), sf.cpu())
    T_used = int(sum(lens))
    o32, sf32 = outs[torch.float32]
    ob, sfb = outs[torch.bfloat16]
    assert torch.all(o32[:, T_used:] == 7.0) and torch.all(ob[:, T_used:] == 7.0), "padding rows were written"
    assert _err(o32[:, :T_used], o_ref[:, :T_used]) <= TOL[dt]
    assert _err(sf32, s_ref) <= TOL[dt]
    assert torch.equal(ob, o32.to(torch.bfloat16))
    assert torch.equal(sfb, sf32)


def test_zero_skip_weights_change_nothing(lib):
    inp = _inputs(1, 3, 200, 128, "gdn", torch.bfloat16, seed=78)
    o_plain, s_plain = _dense(lib, inp, None, torch.float32)
    o_zero, s_zero = _dense(lib, inp, torch.zeros(3, 128), torch.float32)
    assert torch.equal(o_plain, o_zero) and torch.equal(s_plain, s_zero)
