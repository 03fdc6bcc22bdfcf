"""The C-ABI library loads, exports what include/gdn.h declares, and validates
arguments on the host (these calls return before any CUDA work, so no GPU is needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdn.h")


@pytest.fixture(scope="module")
def lib():
    from gated_deltanet_sequence_b200 import build
    build.build()
    from gated_deltanet_sequence_b200 import _lib
    return _lib


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    names = _declared_functions()
    for want in ("lin_attn_chunk_fwd", "gdn_chunk_fwd", "lin_attn_chunk_fwd_varlen", "gdn_chunk_fwd_varlen",
                 "lin_attn_chunk_fwd_ex", "gdn_chunk_fwd_ex", "gdn_decode_step", "gdn_decode_step_ex",
                 "gdn_status_str", "gdn_sync_status", "gdn_set_wait_limit_for_testing", "gdn_version",
                 "gdn_chunk_bwd", "gdn_chunk_bwd_workspace_bytes", "gdn_state_compose", "gdn_state_identity",
                 "gdn_chunk_fwd_host", "gdn_chunk_fwd_host_staging_bytes"):
        assert want in names


def test_library_exports_every_declared_symbol(lib):
    raw = ctypes.CDLL(lib.LIB_PATH)
    for name in _declared_functions():
        assert hasattr(raw, name), f"libgdn.so does not export {name}"


def test_debug_library_exports_the_same_symbols(lib):
    # the bounds-checked build (python -m gated_deltanet_sequence_b200.build --debug-bounds)
    path = os.path.join(os.path.dirname(lib.LIB_PATH), "libgdn_debug.so")
    if not os.path.exists(path):
        pytest.skip("libgdn_debug.so is not built")
    raw = ctypes.CDLL(path)
    for name in lib.EXPORTS:
        assert hasattr(raw, name), f"libgdn_debug.so does not export {name}"
    raw.gdn_status_str.argtypes = [ctypes.c_int]
    raw.gdn_status_str.restype = ctypes.c_char_p
    assert raw.gdn_status_str(6) == b"GDN_ERR_BOUNDS"


def test_status_strings_and_version(lib):
    assert lib.status_str(0) == "GDN_OK"
    assert lib.status_str(4) == "GDN_ERR_TIMEOUT"
    assert lib.status_str(5) == "GDN_ERR_NONFINITE"
    assert lib.status_str(6) == "GDN_ERR_BOUNDS"
    assert lib.status_str(99) == "GDN_ERR_UNKNOWN"
    assert lib.gdn_version() >= 100


FAKE = 0x10000  # 16-byte aligned, never dereferenced: validation fails first


def _prefill(lib, fn, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, beta=FAKE, g=None, o=FAKE, s0=None, s_final=None,
             B=1, H=1, L=8, dk=64, dv=64, chunk=64, scale=1.0, dt=1)
    a.update(kw)
    P = ctypes.c_void_p
    if fn == "gdn":
        return lib.lib.gdn_chunk_fwd(P(a["q"]), P(a["k"]), P(a["v"]), P(a["beta"]), P(a["g"]),
                                     P(a["o"]), P(a["s0"]), P(a["s_final"]), a["B"], a["H"],
                                     a["L"], a["dk"], a["dv"], a["chunk"], a["scale"], a["dt"], None)
    return lib.lib.lin_attn_chunk_fwd(P(a["q"]), P(a["k"]), P(a["v"]), P(a["g"]), P(a["o"]),
                                      P(a["s0"]), P(a["s_final"]), a["B"], a["H"], a["L"],
                                      a["dk"], a["dv"], a["chunk"], a["scale"], a["dt"], None)


@pytest.mark.parametrize("fn", ["gdn", "la"])
@pytest.mark.parametrize("kw,want", [
    (dict(B=0), 1), (dict(H=0), 1), (dict(L=-1), 1), (dict(q=None), 1), (dict(o=None), 1),
    (dict(q=FAKE + 2), 1), (dict(o=FAKE + 8), 1), (dict(s0=FAKE + 4), 1), (dict(chunk=0), 1),
    (dict(dt=7), 1), (dict(scale=float("nan")), 1),
    (dict(dk=96), 2), (dict(dv=32), 2), (dict(chunk=65), 2),
])
def test_prefill_rejects_bad_arguments(lib, fn, kw, want):
    assert _prefill(lib, fn, **kw) == want


def test_gdn_requires_beta(lib):
    assert _prefill(lib, "gdn", beta=None) == 1


@pytest.mark.parametrize("kw,want", [
    (dict(N=0), 1), (dict(q=None), 1), (dict(state=FAKE + 4), 1), (dict(dk=32), 2), (dict(dt=3), 1),
])
def test_decode_rejects_bad_arguments(lib, kw, want):
    a = dict(q=FAKE, k=FAKE, v=FAKE, beta=None, g=None, state=FAKE, o=FAKE, N=1, H=1, dk=64,
             dv=64, scale=1.0, dt=1)
    a.update(kw)
    P = ctypes.c_void_p
    st = lib.lib.gdn_decode_step(P(a["q"]), P(a["k"]), P(a["v"]), P(a["beta"]), P(a["g"]),
                                 P(a["state"]), P(a["o"]), a["N"], a["H"], a["dk"], a["dv"],
                                 a["scale"], a["dt"], None)
    assert st == want


def test_binding_raises_on_bad_shapes(lib):
    import torch
    q = torch.zeros(1, 1, 4, 64)
    with pytest.raises(ValueError):
        lib.gdn_chunk_fwd(q, q, torch.zeros(1, 1, 5, 64), torch.zeros(1, 1, 4))


def _varlen(lib, fn, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, beta=FAKE, g=None, o=FAKE, s0=None, s_final=None, cu=FAKE,
             N=2, H=1, T=8, dk=64, dv=64, chunk=64, scale=1.0, dt=1)
    a.update(kw)
    P = ctypes.c_void_p
    if fn == "gdn":
        return lib.lib.gdn_chunk_fwd_varlen(P(a["q"]), P(a["k"]), P(a["v"]), P(a["beta"]), P(a["g"]),
                                            P(a["o"]), P(a["s0"]), P(a["s_final"]), P(a["cu"]), a["N"],
                                            a["H"], a["T"], a["dk"], a["dv"], a["chunk"], a["scale"],
                                            a["dt"], None)
    return lib.lib.lin_attn_chunk_fwd_varlen(P(a["q"]), P(a["k"]), P(a["v"]), P(a["g"]), P(a["o"]),
                                             P(a["s0"]), P(a["s_final"]), P(a["cu"]), a["N"], a["H"],
                                             a["T"], a["dk"], a["dv"], a["chunk"], a["scale"], a["dt"], None)


@pytest.mark.parametrize("fn", ["gdn", "la"])
@pytest.mark.parametrize("kw,want", [
    (dict(N=0), 1), (dict(cu=None), 1), (dict(cu=FAKE + 2), 1), (dict(H=0), 1), (dict(T=-1), 1),
    (dict(q=None), 1), (dict(o=FAKE + 8), 1), (dict(dt=5), 1), (dict(dk=96), 2), (dict(chunk=65), 2),
])
def test_varlen_rejects_bad_arguments(lib, fn, kw, want):
    assert _varlen(lib, fn, **kw) == want


def test_varlen_gdn_requires_beta(lib):
    assert _varlen(lib, "gdn", beta=None) == 1


def test_varlen_binding_checks_shapes(lib):
    import torch
    q = torch.zeros(2, 8, 64)
    cu = torch.tensor([0, 3, 8], dtype=torch.int32)
    with pytest.raises(ValueError):
        lib.gdn_chunk_fwd_varlen(q, q, torch.zeros(2, 9, 64), torch.zeros(2, 8), cu)
    with pytest.raises(TypeError):
        lib.lin_attn_chunk_fwd_varlen(q, q, q, cu.long())


def _ex(lib, fn, out_dtype=0, d_skip=None, g_per_key=0, no_opts=False, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, beta=FAKE, g=None, o=FAKE, s0=None, s_final=None, cu=None,
             B=1, H=1, L=8, dk=64, dv=64, chunk=64, scale=1.0, dt=1)
    a.update(kw)
    P = ctypes.c_void_p
    opts = None if no_opts else ctypes.byref(lib.FwdOpts(out_dtype, d_skip, g_per_key))
    if fn == "gdn":
        return lib.lib.gdn_chunk_fwd_ex(P(a["q"]), P(a["k"]), P(a["v"]), P(a["beta"]), P(a["g"]), P(a["o"]),
                                        P(a["s0"]), P(a["s_final"]), P(a["cu"]), a["B"], a["H"], a["L"],
                                        a["dk"], a["dv"], a["chunk"], a["scale"], a["dt"], opts, None)
    return lib.lib.lin_attn_chunk_fwd_ex(P(a["q"]), P(a["k"]), P(a["v"]), P(a["g"]), P(a["o"]), P(a["s0"]),
                                         P(a["s_final"]), P(a["cu"]), a["B"], a["H"], a["L"], a["dk"], a["dv"],
                                         a["chunk"], a["scale"], a["dt"], opts, None)


@pytest.mark.parametrize("fn", ["gdn", "la"])
@pytest.mark.parametrize("kw,want", [
    (dict(out_dtype=2), 1), (dict(out_dtype=-1), 1), (dict(d_skip=FAKE + 2), 1), (dict(g_per_key=2), 1),
    (dict(B=0), 1), (dict(o=FAKE + 8), 1), (dict(dt=7), 1), (dict(dk=96), 2), (dict(chunk=65), 2),
    (dict(cu=FAKE + 2), 1), (dict(cu=FAKE, B=0), 1), (dict(no_opts=True, q=None), 1),
])
def test_ex_rejects_bad_arguments(lib, fn, kw, want):
    assert _ex(lib, fn, **kw) == want


def test_ex_gdn_requires_beta(lib):
    assert _ex(lib, "gdn", beta=None) == 1
    assert _ex(lib, "gdn", beta=None, cu=FAKE) == 1


def test_binding_checks_output_options(lib):
    import torch
    q = torch.zeros(1, 2, 4, 64)
    with pytest.raises(TypeError):      # o dtype must be fp32 or bf16
        lib.lin_attn_chunk_fwd(q, q, q, out_dtype=torch.float16)
    with pytest.raises(ValueError):     # d_skip is (H, dv)
        lib.lin_attn_chunk_fwd(q, q, q, d_skip=torch.zeros(3, 64))
    with pytest.raises(TypeError):      # d_skip is fp32
        lib.gdn_chunk_fwd(q, q, q, torch.zeros(1, 2, 4), d_skip=torch.zeros(2, 64, dtype=torch.float64))


def test_binding_checks_vector_gate_shape(lib):
    import torch
    q = torch.zeros(1, 2, 4, 64)
    with pytest.raises(ValueError):     # (B, H, L) or (B, H, L, dk)
        lib.lin_attn_chunk_fwd(q, q, q, torch.zeros(1, 2, 4, 32))


@pytest.mark.parametrize("kw,want", [
    (dict(g_per_key=3), 1), (dict(out_dtype=9), 1), (dict(d_skip=FAKE + 2), 1), (dict(N=0), 1), (dict(dk=32), 2),
])
def test_decode_ex_rejects_bad_arguments(lib, kw, want):
    a = dict(q=FAKE, k=FAKE, v=FAKE, beta=None, g=None, state=FAKE, o=FAKE, N=1, H=1, dk=64, dv=64, scale=1.0, dt=1,
             out_dtype=0, d_skip=None, g_per_key=0)
    a.update(kw)
    P = ctypes.c_void_p
    opts = lib.FwdOpts(a["out_dtype"], a["d_skip"], a["g_per_key"])
    st = lib.lib.gdn_decode_step_ex(P(a["q"]), P(a["k"]), P(a["v"]), P(a["beta"]), P(a["g"]), P(a["state"]),
                                    P(a["o"]), a["N"], a["H"], a["dk"], a["dv"], a["scale"], a["dt"],
                                    ctypes.byref(opts), None)
    assert st == want


def test_state_compose_and_identity_validate_on_the_host(lib):
    P = ctypes.c_void_p
    one = 128 * 128 * 4                                  # bytes of one d = 128 state
    mn, n, out = P(FAKE), P(FAKE + 2 * one), P(FAKE + 4 * one)
    compose, identity = lib.lib.gdn_state_compose, lib.lib.gdn_state_identity
    assert compose(mn, n, None, out, 1.0, 1, 96, None) == 2            # d outside {64, 128}
    assert compose(mn, n, None, out, 1.0, -1, 128, None) == 1
    assert compose(mn, n, None, out, 0.0, 1, 128, None) == 1            # lambda 0
    assert compose(mn, n, None, out, float("inf"), 1, 128, None) == 1
    assert compose(mn, n, None, out, 1e-45, 1, 128, None) == 1          # 1 / lambda overflows
    assert compose(None, n, None, out, 1.0, 1, 128, None) == 1
    assert compose(P(FAKE + 4), n, None, out, 1.0, 1, 128, None) == 1   # misaligned
    assert compose(mn, n, P(FAKE + 4 * one + 64), out, 1.0, 1, 128, None) == 1   # s_in overlaps s_out
    assert compose(mn, n, None, P(FAKE + one // 2), 1.0, 1, 128, None) == 1      # s_out overlaps mn
    assert compose(mn, n, None, out, 1.0, 0, 128, None) == 0           # nothing to do
    assert identity(P(FAKE), 1.0, 1, 32, None) == 2
    assert identity(P(FAKE + 8), 1.0, 1, 64, None) == 1
    assert identity(None, 1.0, 1, 64, None) == 1
    assert identity(P(FAKE), float("nan"), 1, 64, None) == 1
    assert identity(P(FAKE), 1.0, 0, 64, None) == 0


def test_host_pipeline_entry_validates_on_the_host(lib):
    P = ctypes.c_void_p
    f = lib.lib.gdn_chunk_fwd_host
    size = lib.lib.gdn_chunk_fwd_host_staging_bytes
    need = size(2, 3, 100, 128, 128, 1, 1, 1, 0, 1)
    assert need > 0 and need % 256 == 0
    assert size(2, 3, 100, 128, 128, 0, 1, 1, 0, 1) == 0                  # group < 1
    args = [P(FAKE)] * 4 + [None, P(FAKE), None, None, P(FAKE), need, 2, 3, 100, 128, 128, 64, 1.0, 1, 1, None]
    a = list(args); a[0] = None
    assert f(*a) == 1                                                       # q missing
    a = list(args); a[13] = 96
    assert f(*a) == 2                                                       # dk outside {64, 128}
    a = list(args); a[12] = 0
    assert f(*a) == 1                                                       # L < 1
    assert f(*args) == 1                  # these host pointers are not page-locked memory
