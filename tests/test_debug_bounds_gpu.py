"""The bounds-checked debug build (libgdn_debug.so, -DGDN_DEBUG_BOUNDS): its kernels check the
index of each thread-side global access of inputs, outputs and states against the extent the
launch implies and report GDN_ERR_BOUNDS instead of making an out-of-range access. On valid
calls it must report nothing and give the release build's results bit for bit: the tensor-core
prefill kernels (one-CTA Gated DeltaNet dense and packed, the head-size-64 direct form, linear
attention, the vector-gate prep and chain kernels, the segmented long-sequence path), the fp32
chunk kernel (dense, vector gates, packed) and three decode steps run in a child process on each
library."""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import sys, torch
sys.path.insert(0, sys.argv[1])
from gated_deltanet_sequence_b200 import _lib as gdn, workloads as W
out = {}
torch.cuda.set_device(0)
inp = W.make_prefill_inputs(4, 16, 200, 128, 128, mode="gdn", in_dtype=torch.bfloat16, s0=True, seed=901, device="cuda")
out["gdn"] = gdn.gdn_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["g"], s0=inp["s0"],
                              s_final=torch.empty_like(inp["s0"]))
out["la"] = gdn.lin_attn_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], s0=inp["s0"],
                                   s_final=torch.empty_like(inp["s0"]))
gv = W.make_gate_per_key((4, 16), 200, 128, seed=902, device="cuda")
out["vec"] = gdn.gdn_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["beta"], gv, s0=inp["s0"],
                               s_final=torch.empty_like(inp["s0"]))
d64 = W.make_prefill_inputs(4, 16, 130, 64, 64, mode="gdn", in_dtype=torch.bfloat16, s0=True, seed=903, device="cuda")
out["d64"] = gdn.gdn_chunk_fwd(d64["q"], d64["k"], d64["v"], d64["beta"], d64["g"], s0=d64["s0"],
                               s_final=torch.empty_like(d64["s0"]))
lens = [0, 1, 64, 65, 130, 300, 7, 191]
vl = W.make_varlen_inputs(lens, 8, 128, 128, mode="gdn", in_dtype=torch.bfloat16, s0=True, seed=904, device="cuda")
out["varlen"] = gdn.gdn_chunk_fwd_varlen(vl["q"], vl["k"], vl["v"], vl["beta"], vl["cu_seqlens"], vl["g"],
                                         s0=vl["s0"], s_final=torch.empty_like(vl["s0"]))
lg = W.make_prefill_inputs(1, 2, 64 * 130 + 17, 128, 128, mode="gdn", in_dtype=torch.bfloat16, s0=True, seed=905,
                           device="cuda")
out["long"] = gdn.gdn_chunk_fwd(lg["q"], lg["k"], lg["v"], lg["beta"], lg["g"], s0=lg["s0"],
                                s_final=torch.empty_like(lg["s0"]))
f32 = W.make_prefill_inputs(2, 3, 150, 128, 64, mode="gdn", in_dtype=torch.float32, s0=True, seed=907, device="cuda")
out["f32"] = gdn.gdn_chunk_fwd(f32["q"], f32["k"], f32["v"], f32["beta"], f32["g"], s0=f32["s0"],
                               s_final=torch.empty_like(f32["s0"]))
gv32 = W.make_gate_per_key((2, 3), 150, 128, seed=908, device="cuda")
out["f32vec"] = gdn.gdn_chunk_fwd(f32["q"], f32["k"], f32["v"], f32["beta"], gv32, s0=f32["s0"],
                                  s_final=torch.empty_like(f32["s0"]))
vl32 = W.make_varlen_inputs([5, 70, 0, 140], 2, 64, 64, mode="gdn", in_dtype=torch.float32, s0=True, seed=909,
                            device="cuda")
out["f32varlen"] = gdn.gdn_chunk_fwd_varlen(vl32["q"], vl32["k"], vl32["v"], vl32["beta"], vl32["cu_seqlens"],
                                            vl32["g"], s0=vl32["s0"], s_final=torch.empty_like(vl32["s0"]))
dec = W.make_decode_inputs(16, 8, 128, 128, 3, seed=906, device="cuda")
state = dec["state"].clone()
outs = []
for t in range(3):
    outs.append(gdn.gdn_decode_step(dec["q"][t], dec["k"][t], dec["v"][t], dec["beta"][t], dec["g"][t], state))
out["decode"] = (torch.stack(outs), state)
status = gdn.gdn_sync_status()
torch.save({"status": status, "lib": gdn.LIB_PATH,
            "out": {k: tuple(t.cpu() for t in v) for k, v in out.items()}}, sys.argv[2])
'''


def _run(tmp_path, debug):
    env = dict(os.environ)
    if debug:
        env["GDN_LIBRARY"] = "debug"
    else:
        env.pop("GDN_LIBRARY", None)
    path = str(tmp_path / ("debug.pt" if debug else "release.pt"))
    subprocess.run([sys.executable, "-c", CHILD, ROOT, path], env=env, check=True, timeout=600)
    return torch.load(path)


def test_debug_build_reports_nothing_and_matches_release(tmp_path):
    if not os.path.exists(os.path.join(ROOT, "gated_deltanet_sequence_b200", "libgdn_debug.so")):
        pytest.fail("libgdn_debug.so is not built (python -m gated_deltanet_sequence_b200.build --debug-bounds)")
    dbg = _run(tmp_path, True)
    rel = _run(tmp_path, False)
    assert dbg["lib"].endswith("libgdn_debug.so") and rel["lib"].endswith("libgdn.so")
    assert dbg["status"] == 0, f"debug build reported status {dbg['status']}"
    assert rel["status"] == 0
    for k in rel["out"]:
        for a, b in zip(dbg["out"][k], rel["out"][k]):
            assert torch.equal(a, b), f"{k}: debug and release builds differ"
