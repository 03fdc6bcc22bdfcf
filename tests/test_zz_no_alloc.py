"""The backward entry point that allocates nothing (gdn_chunk_bwd_noalloc), for callers that
cannot allocate device memory when they run the backward: a plugin interface that hands over
only input and output buffers, or a runtime whose allocator reserved all device memory up
front. It uses a fixed array in the library's static device memory as its workspace.

Called through the C ABI and compared with gdn_chunk_bwd (which takes a caller-allocated
workspace) on two calls in a row (the second runs on the array's leftover contents); the
two must agree within the backward's parity tolerance. This file is collected last, so a run
that stops at its first failure has run every other test before it.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_sequence_b200 import workloads as W

pytestmark = pytest.mark.gpu

GDN_OK, GDN_ERR_UNSUPPORTED = 0, 2
TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-3}


@pytest.fixture(scope="module")
def lib():
    from gated_deltanet_sequence_b200 import _lib
    return _lib


def _noalloc(lib, inp, do, dsf, chunk, scale):
    """gdn_chunk_bwd_noalloc through the C ABI; the outputs are allocated by the test."""
    q, k, v, beta, g, s0 = (inp[n] for n in ("q", "k", "v", "beta", "g", "s0"))
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    f32 = dict(dtype=torch.float32, device="cuda")
    out = {"dq": torch.full((B, H, L, dk), float("nan"), **f32), "dk": torch.full((B, H, L, dk), float("nan"), **f32),
           "dv": torch.full((B, H, L, dv), float("nan"), **f32), "dbeta": torch.full((B, H, L), float("nan"), **f32),
           "dg": torch.full((B, H, L), float("nan"), **f32), "ds0": torch.full((B, H, dk, dv), float("nan"), **f32)}
    P = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    st = lib.lib.gdn_chunk_bwd_noalloc(P(q), P(k), P(v), P(beta), P(g), P(s0), P(do), P(dsf), P(out["dq"]),
                                       P(out["dk"]), P(out["dv"]), P(out["dbeta"]), P(out["dg"]), P(out["ds0"]),
                                       B, H, L, dk, dv, chunk, float(scale), lib._dtype_code(q),
                                       ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, out


@pytest.mark.parametrize("dtype,B,H,dk,dv,L,chunk", [(torch.bfloat16, 1, 2, 128, 128, 300, 64),
                                                   (torch.float32, 2, 3, 64, 128, 150, 32)])
def test_noalloc_backward_matches_the_workspace_backward(lib, dtype, B, H, dk, dv, L, chunk):
    assert lib.gdn_chunk_bwd_workspace_bytes(B, H, L, dk, dv, chunk) <= 16 << 20
    host = W.make_prefill_inputs(B, H, L, dk, dv, mode="gdn", in_dtype=dtype, s0=True, seed=811)
    inp = {n: x.cuda() for n, x in host.items() if x is not None}
    gen = torch.Generator().manual_seed(812)
    do = torch.randn(B, H, L, dv, generator=gen).cuda()
    dsf = torch.randn(B, H, dk, dv, generator=gen).cuda()
    ref = lib.gdn_chunk_bwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["g"], do, s0=inp["s0"], ds_final=dsf,
                            chunk=chunk, scale=0.9)
    for call in range(2):
        st, got = _noalloc(lib, inp, do, dsf, chunk, 0.9)
        assert st == GDN_OK, lib.status_str(st)
        assert lib.gdn_sync_status() == GDN_OK
        for name, r in ref.items():
            err = oracle.max_norm_err(got[name].cpu(), r.cpu())
            assert np.isfinite(err) and err <= TOL[dtype], f"call {call} {name}: {err:.3e}"


def test_noalloc_rejects_a_call_beyond_its_array(lib):
    B, H, L, d = 3, 1, 4096, 128          # 3 heads x 128 states of 64 KB = 24 MiB > 16 MiB
    assert lib.gdn_chunk_bwd_workspace_bytes(B, H, L, d, d, 64) > 16 << 20
    # buffers of the full sizes, so that the call would stay in bounds even if it ran
    f32 = dict(dtype=torch.float32, device="cuda")
    qkv = torch.zeros(3, B, H, L, d, dtype=torch.bfloat16, device="cuda")
    tok = torch.zeros(B, H, L, d, **f32)
    grads = torch.zeros(3, B, H, L, d, **f32)
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    st = lib.lib.gdn_chunk_bwd_noalloc(P(qkv[0]), P(qkv[1]), P(qkv[2]), None, None, None, P(tok), None,
                                       P(grads[0]), P(grads[1]), P(grads[2]), None, None, None, B, H, L, d, d,
                                       64, 1.0, 1, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == GDN_ERR_UNSUPPORTED
    assert lib.gdn_sync_status() == GDN_OK
