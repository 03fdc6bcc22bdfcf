"""The host-buffer prefill (copies in groups of sequences, overlapped with compute on
three streams) gives exactly the bits of one device call on the whole batch."""
import pytest
import torch

from gated_deltanet_sequence_b200 import workloads as W


def test_requires_pinned_host_tensors():
    from gated_deltanet_sequence_b200.host import gdn_chunk_fwd_host
    q = torch.zeros(2, 1, 8, 64)
    with pytest.raises(ValueError):
        gdn_chunk_fwd_host(q, q, q, torch.zeros(2, 1, 8))


@pytest.mark.gpu
@pytest.mark.parametrize("group,s0,gated", [(1, False, True), (3, True, True), (8, True, False), (2, False, True)])
def test_host_pipeline_matches_device_call(group, s0, gated):
    from gated_deltanet_sequence_b200 import _lib
    from gated_deltanet_sequence_b200.host import gdn_chunk_fwd_host
    inp = W.make_prefill_inputs(7, 4, 300, 128, 128, mode="gdn", in_dtype=torch.bfloat16, s0=s0, seed=110)
    if not gated:
        inp["g"] = None
    pin = {n: (None if t is None else t.pin_memory()) for n, t in inp.items()}
    o, sf = gdn_chunk_fwd_host(pin["q"], pin["k"], pin["v"], pin["beta"], pin["g"], s0=pin["s0"], s_final=True,
                               group=group)
    torch.cuda.current_stream().synchronize()
    assert _lib.gdn_sync_status() == 0
    dev = {n: (None if t is None else t.cuda()) for n, t in inp.items()}
    o_ref, sf_ref = _lib.gdn_chunk_fwd(dev["q"], dev["k"], dev["v"], dev["beta"], dev["g"], s0=dev["s0"],
                                       s_final=torch.empty(7, 4, 128, 128, device="cuda"))
    assert torch.equal(o, o_ref.cpu()) and torch.equal(sf, sf_ref.cpu())
