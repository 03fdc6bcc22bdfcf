"""Failure path of the tensor-core kernels: a bounded wait that gives up.

The wait limit is lowered to a few hundred clock cycles (gdn_set_wait_limit_for_testing),
far below the time a TMA tile load from HBM takes, so the first waits of every CTA give
up while the work they wait for is still legitimately in flight. Nothing is broken on
purpose and nothing hangs: the kernel stops issuing, drains the copies and tensor-core
products it has issued, frees its tensor memory and returns; gdn_sync_status reports
GDN_ERR_TIMEOUT. The next call with the default limit must then be clean and match the
oracle (the context stays usable). Covers the one-CTA and cluster forms of the Gated
DeltaNet kernel, the linear-attention kernel, and the prep and chain kernels (vector-valued
gates; and a long sequence over few heads, where they run in segments on two streams).
"""
import pytest
import torch

import oracle
from gated_deltanet_sequence_b200 import workloads as W

pytestmark = pytest.mark.gpu

GDN_OK, GDN_ERR_TIMEOUT = 0, 4


@pytest.fixture(scope="module")
def lib():
    from gated_deltanet_sequence_b200 import _lib
    yield _lib
    _lib.gdn_set_wait_limit_for_testing(0)


# (entry, B, H, L, vector gates): 4 x 16 heads take the one-CTA form (3 x 64 CTAs exceed the
# SM count), 1 x 2 heads the cluster form; vector gates the prep and chain kernels; 130 chunks
# over 2 heads the segmented prep and chain kernels
CASES = {"gdn_one_cta": ("gdn", 4, 16, 200, False), "gdn_cluster": ("gdn", 1, 2, 200, False),
         "lin_attn": ("la", 1, 2, 200, False), "gdn_vector_gate": ("gdn", 1, 2, 200, True),
         "gdn_long_segments": ("gdn", 1, 2, 64 * 130, False)}


def _run(lib, entry, inp, o, sf):
    q, k, v, beta, g = (inp[n].cuda() for n in ("q", "k", "v", "beta", "g"))
    if entry == "gdn":
        lib.gdn_chunk_fwd(q, k, v, beta, g, o=o, s_final=sf)
    else:
        lib.lin_attn_chunk_fwd(q, k, v, g, o=o, s_final=sf)


@pytest.mark.parametrize("case", list(CASES))
def test_wait_gives_up_then_next_call_is_clean(lib, case):
    entry, B, H, L, vector = CASES[case]
    d = 128
    inp = W.make_prefill_inputs(B, H, L, d, d, mode="gdn", in_dtype=torch.bfloat16, seed=606)
    if vector:
        inp["g"] = W.make_gate_per_key((B, H), L, d, seed=607)
    o = torch.empty(B, H, L, d, device="cuda")
    sf = torch.empty(B, H, d, d, device="cuda")
    for _ in range(3):                          # nothing pending from earlier tests
        if lib.gdn_sync_status() == GDN_OK:
            break
    assert lib.gdn_sync_status() == GDN_OK
    lib.gdn_set_wait_limit_for_testing(300)
    try:
        _run(lib, entry, inp, o, sf)
        assert lib.gdn_sync_status() == GDN_ERR_TIMEOUT
    finally:
        lib.gdn_set_wait_limit_for_testing(0)
    assert lib.gdn_sync_status() == GDN_OK      # the condition was reported once
    o.fill_(float("nan"))
    sf.fill_(float("nan"))
    _run(lib, entry, inp, o, sf)
    assert lib.gdn_sync_status() == GDN_OK
    beta = inp["beta"] if entry == "gdn" else None
    o_ref, s_ref = oracle.recurrent_fwd(inp["q"], inp["k"], inp["v"], beta, inp["g"])
    assert oracle.max_norm_err(o.cpu(), o_ref) <= 2e-3
    assert oracle.max_norm_err(sf.cpu(), s_ref) <= 2e-3
