"""GPU parity of the sequence-split (context-parallel) prefill against the fp64 oracle.

The composition kernel (gdn_state_compose) and the identity states are checked through the
C ABI against plain fp64 products; ``segmented_prefill`` (the split run on one device, the
segments as sequences of packed launches) against one oracle run of the whole sequence, for
every mode, small cases spanning several chunks and a ragged tail, and the long-context
workload (1 x 32 heads x 65 536 tokens, s0 != 0) split into 4 segments on sampled heads.
Error metric and bounds as in the other parity tests: max|x - ref| / max|ref|, 2e-3 for bf16
inputs, 1e-5 for fp32.
"""
import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_sequence_b200 import workloads as W

pytestmark = pytest.mark.gpu

MODES = {"plain": (False, False), "gated": (False, True), "delta": (True, False), "gdn": (True, True)}


@pytest.fixture(scope="module")
def cp():
    from gated_deltanet_sequence_b200 import _lib, context_parallel
    return _lib, context_parallel


def _inputs(H, L, d, mode, dtype, seed):
    delta, gated = MODES[mode]
    inp = W.make_prefill_inputs(1, H, L, d, d, mode="gdn", in_dtype=dtype, s0=True, seed=seed)
    if not delta:
        inp["beta"] = None
    if not gated:
        inp["g"] = None
    return inp


def _check(x, ref, tol, what):
    err = oracle.max_norm_err(x, ref)
    assert np.isfinite(err) and err <= tol, f"{what}: max-normalised error {err:.3e} > {tol:.1e}"


@pytest.mark.parametrize("d,count", [(128, 5), (64, 3)])
def test_compose_and_identity_kernels(cp, d, count):
    lib, _ = cp
    gen = torch.Generator().manual_seed(d + count)
    mn, n, s_in = (torch.randn(count, d, d, generator=gen) for _ in range(3))
    out = torch.full((count, d, d), float("nan"), device="cuda")
    lib.gdn_state_compose(mn.cuda(), n.cuda(), s_in.cuda(), out, 256.0)
    ref = np.einsum("cij,cjk->cik", (mn - n).double().numpy() / 256.0, s_in.double().numpy()) + n.double().numpy()
    _check(out.cpu(), ref, 1e-5, "compose")
    lib.gdn_state_compose(mn.cuda(), n.cuda(), None, out)       # s_in NULL: the zero state
    assert torch.equal(out.cpu(), n)
    eye = torch.full((count, d, d), float("nan"), device="cuda")
    lib.gdn_state_identity(eye, 256.0)
    assert torch.equal(eye.cpu(), 256.0 * torch.eye(d).repeat(count, 1, 1))
    assert lib.gdn_sync_status() == 0


@pytest.mark.parametrize("mode", list(MODES))
@pytest.mark.parametrize("L,segments", [(700, 4), (300, 3), (129, 2), (64, 4)])
def test_segmented_prefill_bf16_d128(cp, mode, L, segments):
    lib, ctx = cp
    inp = _inputs(3, L, 128, mode, torch.bfloat16, seed=40 + L + segments)
    dev = {n: (None if x is None else x.cuda()) for n, x in inp.items()}
    o, sf = ctx.segmented_prefill(dev["q"], dev["k"], dev["v"], dev["beta"], dev["g"], dev["s0"],
                                  segments=segments)
    assert lib.gdn_sync_status() == 0
    o_ref, s_ref = oracle.recurrent_fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["g"], inp["s0"])
    _check(o.cpu(), o_ref, 2e-3, f"o {mode} L={L} P={segments}")
    _check(sf.cpu(), s_ref, 2e-3, f"S {mode} L={L} P={segments}")


@pytest.mark.parametrize("mode", ["gdn", "plain"])
def test_segmented_prefill_fp32_d64_uneven_bounds(cp, mode):
    lib, ctx = cp
    L = 333
    inp = _inputs(2, L, 64, mode, torch.float32, seed=77)
    dev = {n: (None if x is None else x.cuda()) for n, x in inp.items()}
    o, sf = ctx.segmented_prefill(dev["q"], dev["k"], dev["v"], dev["beta"], dev["g"], dev["s0"],
                                  bounds=[0, 5, 130, 131, 260, L], chunk=32)
    assert lib.gdn_sync_status() == 0
    o_ref, s_ref = oracle.recurrent_fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["g"], inp["s0"])
    _check(o.cpu(), o_ref, 1e-5, f"o {mode}")
    _check(sf.cpu(), s_ref, 1e-5, f"S {mode}")


def test_segmented_long_context_workload_sampled(cp):
    # the long-context workload as the benchmark's split row runs it: 4 segments of 16 384 tokens
    lib, ctx = cp
    w = W.WORKLOADS[3]
    inp = W.make_workload_inputs(w, device="cuda")
    o, sf = ctx.segmented_prefill(inp["q"], inp["k"], inp["v"], inp["beta"], inp["g"], inp["s0"], segments=4)
    assert lib.gdn_sync_status() == 0
    assert torch.isfinite(o).all() and torch.isfinite(sf).all()
    heads = [0, 17, 31]
    sel = lambda x: x[0, heads].cpu()
    o_ref, s_ref = oracle.recurrent_fwd(sel(inp["q"]), sel(inp["k"]), sel(inp["v"]), sel(inp["beta"]),
                                        sel(inp["g"]), sel(inp["s0"]))
    _check(sel(o), o_ref, 2e-3, "o long split")
    _check(sel(sf), s_ref, 2e-3, "S long split")
