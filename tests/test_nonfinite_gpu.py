"""Non-finite results of the tensor-core prefill kernels are reported, not silent.

Those kernels take fp16 UMMA operands (10-bit mantissa, largest finite value 65504). A
call whose values leave that range stores inf / NaN in o or S_final; the kernels then
record the condition in the device-side word and the next gdn_sync_status returns
GDN_ERR_NONFINITE (once). Here v is scaled to about 3e5, which is exact in bf16 but beyond
the fp16 range, on the one-CTA and cluster forms of the Gated DeltaNet kernel, on the
linear-attention kernel, and on the prep and chain kernels (vector-valued gates; a long
sequence over few heads in segments); the same call with the values in range must then
report GDN_OK.
"""
import pytest
import torch

from gated_deltanet_sequence_b200 import workloads as W

pytestmark = pytest.mark.gpu

GDN_OK, GDN_ERR_NONFINITE = 0, 5

# (entry, B, H, L, vector gates): 64 heads take the one-CTA form, 2 heads the cluster form;
# vector gates the prep and chain kernels, 130 chunks over 2 heads the segmented ones
CASES = {"gdn_one_cta": ("gdn", 1, 64, 150, False), "gdn_cluster": ("gdn", 1, 2, 150, False),
         "lin_attn": ("la", 1, 2, 150, False), "gdn_vector_gate": ("gdn", 1, 2, 150, True),
         "gdn_long_segments": ("gdn", 1, 2, 64 * 130, False)}


@pytest.fixture(scope="module")
def lib():
    from gated_deltanet_sequence_b200 import _lib
    return _lib


def _run(lib, entry, inp, v_scale):
    q, k, beta, g = (inp[n].cuda() for n in ("q", "k", "beta", "g"))
    v = (inp["v"].float() * v_scale).to(torch.bfloat16).cuda()
    if entry == "gdn":
        o, sf = lib.gdn_chunk_fwd(q, k, v, beta, g, s_final=torch.empty(q.shape[0], q.shape[1], 128, 128,
                                                                        device="cuda"))
    else:
        o, sf = lib.lin_attn_chunk_fwd(q, k, v, g, s_final=torch.empty(q.shape[0], q.shape[1], 128, 128,
                                                                       device="cuda"))
    return o, sf


@pytest.mark.parametrize("case", list(CASES))
def test_out_of_range_values_are_reported(lib, case):
    entry, B, H, L, vector = CASES[case]
    inp = W.make_prefill_inputs(B, H, L, 128, 128, mode="gdn", in_dtype=torch.bfloat16, seed=909)
    if vector:
        inp["g"] = W.make_gate_per_key((B, H), L, 128, seed=910)
    for _ in range(3):                          # nothing pending from earlier tests
        if lib.gdn_sync_status() == GDN_OK:
            break
    assert lib.gdn_sync_status() == GDN_OK
    o, sf = _run(lib, entry, inp, 3.0e5)
    assert lib.gdn_sync_status() == GDN_ERR_NONFINITE
    assert not (torch.isfinite(o).all() and torch.isfinite(sf).all())
    assert lib.gdn_sync_status() == GDN_OK      # reported once
    o, sf = _run(lib, entry, inp, 1.0)
    assert lib.gdn_sync_status() == GDN_OK
    assert torch.isfinite(o).all() and torch.isfinite(sf).all()
