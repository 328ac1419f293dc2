"""C-ABI checks that need no GPU: the library loads, exports every function
that include/gdn.h declares, and rejects bad arguments on the host before
any CUDA call (fake pointers are never dereferenced on these paths)."""
import ctypes
import os
import re

import pytest

from gated_delta_rule_72_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdn.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"GDN_API\s+[\w\s\*]+?\b(gdn_\w+)\s*\(", text)))


def test_header_declares_entry_points():
    names = _declared()
    for required in ("gdn_scan_causal", "gdn_scan_bidir", "gdn_step", "gdn_workspace_size",
                     "gdn_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name
    assert set(_declared()) <= set(_lib.SIGNATURES)


def test_exports_nothing_undeclared():
    out = os.popen("nm -D --defined-only %s" % _lib.LIB_PATH).read()
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    assert exported == set(_declared())


def test_status_strings(lib):
    for code in _lib.STATUS:
        s = _lib.gdn_status_string(code)
        assert s and s != "unknown status"
    assert _lib.gdn_status_string(12345) == "unknown status"
    assert "sm_100a" in _lib.gdn_version()


def test_workspace_size_rules(lib):
    assert _lib.gdn_workspace_size(1, 0, 2, 64, 64, 0, 0, 0) == 0          # T = 0: nothing
    assert _lib.gdn_workspace_size(1, 256, 2, 96, 64, 0, 0, 0) == 0        # unsupported dk
    assert _lib.gdn_workspace_size(0, 256, 2, 64, 64, 0, 0, 0) == 0        # B < 1
    assert _lib.gdn_workspace_size(1, 256, 2, 64, 64, 7, 0, 0) == 0        # bad dtype
    assert _lib.gdn_workspace_size(1, 256, 2, 64, 64, 0, 9, 0) == 0        # bad output dtype
    a = _lib.gdn_workspace_size(1, 256, 2, 64, 64, 0, 0, 0)
    b = _lib.gdn_workspace_size(1, 256, 2, 64, 64, 0, 0, 1)
    assert a > 0 and b > a and a % 256 == 0 and b % 256 == 0
    # bf16 inputs, bf16 output, bidirectional: an fp32 partial output is kept
    big = _lib.gdn_workspace_size(1, 75600, 20, 128, 128, 1, 1, 1)
    assert big >= 75600 * 20 * 128 * 4


FAKE = 0x10000  # 16-byte aligned, never dereferenced on the rejected paths


def _causal(**kw):
    args = dict(q=FAKE, k=FAKE, v=FAKE, alpha=FAKE, beta=FAKE, state_in=None, state_out=None,
                o=FAKE, B=1, T=64, H=2, dk=64, dv=64, dt=0, o_dt=0, workspace=FAKE, ws_bytes=1 << 40,
                stream=None)
    args.update(kw)
    return _lib.gdn_scan_causal(*args.values())


def test_rejects_before_launch(lib):
    assert _causal(q=None) == -1
    assert _causal(o=None) == -1
    assert _causal(B=0) == -2
    assert _causal(H=0) == -2
    assert _causal(T=-1) == -2
    assert _causal(dt=5) == -3
    assert _causal(o_dt=-1) == -3
    assert _causal(k=FAKE + 4) == -4
    assert _causal(o=FAKE + 8) == -4
    assert _causal(alpha=FAKE + 2) == -4
    assert _causal(alpha=FAKE + 4, beta=FAKE + 8, ws_bytes=100) == -6  # gates need 4 bytes only
    assert _causal(state_in=FAKE + 2) == -4
    assert _causal(dk=96) == -5
    assert _causal(dv=32) == -5
    assert _causal(workspace=None) == -1
    assert _causal(workspace=FAKE + 16) == -4        # workspace needs 256-byte alignment
    assert _causal(ws_bytes=100) == -6
    # state_in and state_out that overlap without being equal
    assert _causal(state_in=FAKE, state_out=FAKE + 256) == -2


def test_step_requires_state(lib):
    st = _lib.gdn_step(FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, 1, 64, 2, 64, 64, 0, 0, FAKE,
                       1 << 40, None)
    assert st == -1


def test_bidir_rejects(lib):
    st = _lib.gdn_scan_bidir(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 64, 2, 64, 128, 1, 0, FAKE, 10,
                             None)
    assert st == -6
    st = _lib.gdn_scan_bidir(FAKE, None, FAKE, FAKE, FAKE, FAKE, 1, 64, 2, 64, 128, 1, 0, FAKE,
                             1 << 40, None)
    assert st == -1


def test_empty_scan_without_state_is_a_noop(lib):
    # T = 0, no state buffers: nothing to do, no CUDA call is made
    assert _causal(T=0, q=None, k=None, v=None, alpha=None, beta=None, o=None, workspace=None,
                   ws_bytes=0) == 0


def test_python_api_refuses_cpu_tensors():
    import torch
    import gated_delta_rule_72_b200 as g
    x = torch.zeros(1, 8, 1, 64)
    a = torch.ones(1, 8, 1)
    with pytest.raises(ValueError, match="CUDA"):
        g.scan_causal(x, x, x, a, a)
    with pytest.raises(ValueError, match="CUDA"):
        g.scan_bidir(x, x, x, a, a)


def test_noalloc_rejects_oversized_before_launch(lib):
    """gdn_step_noalloc refuses work whose scratch would exceed its fixed
    array, before touching the GPU (fake pointers are never used)."""
    B, T, H, d = 1, 64 * 2000, 16, 128      # fp32 inputs: the CUDA-core path needs scratch
    assert _lib.gdn_workspace_size(B, T, H, d, d, 0, 0, 0) > _lib.GDN_NOALLOC_SCRATCH_BYTES
    st = _lib.gdn_step_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, B, T, H, d, d, 0, 0, None)
    assert st == -6
    st = _lib.gdn_step_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, 1, 64, 2, 64, 64, 0, 0, None)
    assert st == -1
    st = _lib.gdn_step_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 64, 2, 96, 64, 0, 0, None)
    assert st == -5


def test_short_call_threshold_is_clamped(lib):
    """gdn_set_short_call_tokens: negative = automatic (-1, the default), else
    clamped to at most 64; returns the previous setting (host-side only)."""
    prev = lib.gdn_set_short_call_tokens(1000)
    try:
        assert lib.gdn_set_short_call_tokens(-5) == 64
        assert lib.gdn_set_short_call_tokens(0) == -1
        assert lib.gdn_set_short_call_tokens(17) == 0
        assert lib.gdn_set_short_call_tokens(17) == 17
    finally:
        lib.gdn_set_short_call_tokens(prev)


def test_chain_segment_setting_round_trips(lib):
    """gdn_set_chain_segments: values below 1 mean automatic (-1, the
    default); returns the previous setting (host-side only)."""
    prev = lib.gdn_set_chain_segments(4)
    try:
        assert lib.gdn_set_chain_segments(0) == 4
        assert lib.gdn_set_chain_segments(-3) == -1
        assert lib.gdn_set_chain_segments(7) == -1
        assert lib.gdn_set_chain_segments(7) == 7
    finally:
        lib.gdn_set_chain_segments(prev)


def _bidir_states(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, alpha=FAKE, beta=FAKE, state_in=None, state_in_bwd=None,
             state_out=None, state_out_bwd=None, o=FAKE, B=1, T=64, H=2, dk=64, dv=64, dt=0, o_dt=0,
             workspace=FAKE, ws_bytes=10, stream=None)
    a.update(kw)
    return _lib.gdn_scan_bidir_states(*a.values())


def test_bidir_states_rejects_before_launch(lib):
    """Overlap and alignment rules of the four state buffers, checked before
    the workspace size (ws_bytes=10 would otherwise give -6)."""
    S = 1 << 16                      # bytes of one state: 1*2*64*64*4 = 32 KB < 64 KB apart
    A, Bb, C, D = FAKE, FAKE + S, FAKE + 2 * S, FAKE + 3 * S
    assert _bidir_states(state_in=A + 4) == -4
    assert _bidir_states(state_out_bwd=D + 8) == -4
    # both outputs in one buffer, or an output over the other direction's input
    assert _bidir_states(state_out=C, state_out_bwd=C) == -2
    assert _bidir_states(state_in=A, state_out_bwd=A) == -2
    assert _bidir_states(state_in_bwd=Bb, state_out=Bb + 256) == -2
    # each direction in place, or four separate buffers: only the workspace is short
    assert _bidir_states(state_in=A, state_out=A, state_in_bwd=Bb, state_out_bwd=Bb) == -6
    assert _bidir_states(state_in=A, state_in_bwd=Bb, state_out=C, state_out_bwd=D) == -6


def _readout(**kw):
    a = dict(o=FAKE, o_dt=0, z=FAKE, z_dt=0, gamma=None, eps=1e-6, y=FAKE + (1 << 20), y_dt=0, B=1, T=8, H=2,
             dv=64, stream=None)
    a.update(kw)
    return _lib.gdn_readout_gate(*a.values())


def test_readout_rejects_before_launch(lib):
    """gdn_readout_gate argument checks (no CUDA call on these paths)."""
    assert _readout(o_dt=3) == -3
    assert _readout(y_dt=-1) == -3
    assert _readout(dv=96) == -5
    assert _readout(B=0) == -2
    assert _readout(eps=-1.0) == -2
    assert _readout(eps=float("nan")) == -2
    assert _readout(o=None) == -1
    assert _readout(z=FAKE + 8) == -4
    assert _readout(gamma=FAKE + 2) == -4
    # y over part of o, or over o with another dtype
    assert _readout(y=FAKE + 256) == -2
    assert _readout(y=FAKE, y_dt=1) == -2
    # T = 0: nothing to do, no pointer needed
    assert _readout(T=0, o=None, z=None, y=None) == 0


def _vda(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, alpha_frame=FAKE, beta=FAKE, state_in=None, state_in_bwd=None,
             state_out=None, state_out_bwd=None, o=FAKE, B=1, F=3, U=40, H=2, dk=128, dv=128, bidir=1, dt=1,
             o_dt=0, workspace=FAKE, ws_bytes=10, stream=None)
    a.update(kw)
    return _lib.gdn_vda_scan(*a.values())


def test_vda_rejects_before_launch(lib):
    """gdn_vda_scan argument checks (no CUDA call on these paths)."""
    assert _vda(U=0) == -2
    assert _vda(F=-1) == -2
    assert _vda(dk=96) == -5
    assert _vda(dt=7) == -3
    assert _vda(q=None) == -1
    assert _vda(k=FAKE + 8) == -4
    assert _vda(state_in=FAKE + 4) == -4
    assert _vda(state_out=FAKE + (1 << 20), state_out_bwd=FAKE + (1 << 20)) == -2   # both outputs in one buffer
    assert _vda() == -6                                    # workspace too small
    need = lib.gdn_vda_workspace_size(1, 3, 40, 2, 128, 128, 1)
    # A and B per frame-head (64 KB each at d = 128), the two directions' states
    assert need == 3 * 2 * (65536 + 65536) + 2 * 3 * 2 * 65536
    assert lib.gdn_vda_workspace_size(1, 0, 40, 2, 128, 128, 1) == 0
    assert lib.gdn_vda_workspace_size(1, 3, 0, 2, 128, 128, 1) == 0
    # no frames: nothing to do, no pointer needed
    assert _vda(F=0, q=None, k=None, v=None, alpha_frame=None, beta=None, o=None, workspace=None) == 0


def test_python_api_refuses_cpu_tensors_for_new_calls():
    import torch
    import gated_delta_rule_72_b200 as gdn
    q = torch.zeros(1, 6, 1, 64)
    a = torch.ones(1, 6, 1)
    with pytest.raises(ValueError):
        gdn.vda_scan(q, q, q, torch.ones(1, 2, 1), a, 3)
    with pytest.raises(ValueError):
        gdn.vda_scan(q, q, q, torch.ones(1, 2, 1), a, 4)   # T = 6 is not a multiple of U = 4
    with pytest.raises(ValueError):
        gdn.readout_gate(q, q)


def _declared_arity():
    """Parameter count of every GDN_API function in the header."""
    text = open(HEADER).read()
    out = {}
    for m in re.finditer(r"GDN_API\s+[\w\s\*]+?\b(gdn_\w+)\s*\(([^)]*)\)\s*;", text):
        params = m.group(2).strip()
        out[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_signatures_match_the_header():
    """The ctypes binding passes exactly as many arguments as each C function
    declares (a missing or extra argument would shift every later one)."""
    arity = _declared_arity()
    assert set(arity) == set(_lib.SIGNATURES), set(arity) ^ set(_lib.SIGNATURES)
    for name, (_, argtypes) in _lib.SIGNATURES.items():
        assert len(argtypes) == arity[name], (name, len(argtypes), arity[name])


def test_binding_argument_types_match_the_header():
    """Each argument's ctypes type fits its C type: pointers as pointers,
    int and enum as c_int, size_t as c_size_t, float as c_float."""
    text = open(HEADER).read()
    for m in re.finditer(r"GDN_API\s+[\w\s\*]+?\b(gdn_\w+)\s*\(([^)]*)\)\s*;", text):
        name, params = m.group(1), m.group(2).strip()
        if params in ("", "void"):
            continue
        argtypes = _lib.SIGNATURES[name][1]
        for decl, ct in zip([p.strip() for p in params.split(",")], argtypes):
            if "*" in decl:
                assert ct is ctypes.c_void_p or issubclass(ct, (ctypes._Pointer, ctypes.c_char_p)), (name, decl, ct)
            elif decl.startswith("size_t"):
                assert ct is ctypes.c_size_t, (name, decl, ct)
            elif decl.startswith("float"):
                assert ct is ctypes.c_float, (name, decl, ct)
            else:
                assert decl.split()[0] in ("int", "gdn_dtype", "gdn_status"), (name, decl)
                assert ct is ctypes.c_int, (name, decl, ct)
