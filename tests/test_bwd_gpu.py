"""GPU parity of the backward pass (gdn_chunk_bwd) against the oracle's gradients (fp64
autograd of the token recurrence; page "混合注意力学习(1)", section "Transformers 就是
RNNs": the gradients on the full training sequence follow from the chain rule through the
recurrence). Every gradient is compared as a whole tensor with the max-normalised error:
1e-4 for fp32 inputs (the kernel accumulates in fp32 over the whole sequence) and 2e-3
for bf16 inputs; the inputs are the same bf16-rounded values on both sides."""
import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_sequence_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-3}
MODES = {"plain": (False, False), "gated": (False, True), "delta": (True, False), "gdn": (True, True)}


@pytest.fixture(scope="module")
def lib():
    from gated_deltanet_sequence_b200 import _lib
    return _lib


def _check(x, ref, tol, what):
    err = oracle.max_norm_err(x, ref)
    assert np.isfinite(err) and err <= tol, f"{what}: max-normalised error {err:.3e} > {tol:.1e}"


@pytest.mark.parametrize("mode", list(MODES))
@pytest.mark.parametrize("dk,dv,dtype,L,chunk", [(64, 64, torch.float32, 150, 64), (128, 128, torch.bfloat16, 200, 64),
                                                 (64, 128, torch.float32, 77, 16), (128, 64, torch.bfloat16, 65, 128)])
def test_gradients_match_the_oracle(lib, mode, dk, dv, dtype, L, chunk):
    delta, gated = MODES[mode]
    B, H = 2, 2
    inp = W.make_prefill_inputs(B, H, L, dk, dv, mode="gdn", in_dtype=dtype, s0=True, seed=707 + L)
    gen = torch.Generator().manual_seed(708 + L)
    do = torch.randn(B, H, L, dv, generator=gen)
    dsf = torch.randn(B, H, dk, dv, generator=gen)
    beta = inp["beta"] if delta else None
    g = inp["g"] if gated else None
    dev = lambda x: None if x is None else x.cuda()
    gr = lib.gdn_chunk_bwd(dev(inp["q"]), dev(inp["k"]), dev(inp["v"]), dev(beta), dev(g), dev(do), s0=dev(inp["s0"]),
                           ds_final=dev(dsf), chunk=chunk, scale=0.8)
    assert lib.gdn_sync_status() == 0
    _, _, ref = oracle.recurrent_bwd(inp["q"], inp["k"], inp["v"], beta, g, inp["s0"], do=do, ds_final=dsf, scale=0.8)
    for name in ("dq", "dk", "dv", "dbeta", "dg", "ds0"):
        if ref[name] is None:
            assert gr[name] is None
            continue
        _check(gr[name].cpu(), ref[name], TOL[dtype], f"{mode} {name}")


def test_gradients_do_not_depend_on_the_chunk(lib):
    inp = W.make_prefill_inputs(1, 2, 130, 64, 64, mode="gdn", in_dtype=torch.float32, s0=True, seed=709)
    do = torch.randn(1, 2, 130, 64, generator=torch.Generator().manual_seed(710)).cuda()
    d = {n: x.cuda() for n, x in inp.items() if x is not None}
    a = lib.gdn_chunk_bwd(d["q"], d["k"], d["v"], d["beta"], d["g"], do, s0=d["s0"], chunk=64)
    b = lib.gdn_chunk_bwd(d["q"], d["k"], d["v"], d["beta"], d["g"], do, s0=d["s0"], chunk=7)
    for name in a:
        assert torch.equal(a[name], b[name]), name   # the same token arithmetic, recomputed differently


def test_workspace_too_small_is_rejected(lib):
    inp = W.make_prefill_inputs(1, 1, 64, 64, 64, mode="gdn", in_dtype=torch.float32, seed=711)
    d = {n: x.cuda() for n, x in inp.items() if x is not None}
    need = lib.gdn_chunk_bwd_workspace_bytes(1, 1, 64, 64, 64, 64)
    ws = torch.empty(need - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(lib.GdnError):
        lib.gdn_chunk_bwd(d["q"], d["k"], d["v"], d["beta"], d["g"], torch.zeros(1, 1, 64, 64, device="cuda"),
                          workspace=ws)
