"""C-ABI checks that need no GPU: the library loads, exports every function the
header declares, and rejects bad arguments synchronously, before any CUDA call.

Fake device addresses are used only for calls that must fail validation; no
call here reaches a kernel launch.
"""

import ctypes
import os
import re

import pytest

import hybrid_linear_attention_frame_b200 as G
from hybrid_linear_attention_frame_b200 import gdn as B

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "gdn.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(gdn_\w+)\s*\(", src, flags=re.M)))


def test_library_loads_and_exports_header_symbols():
    lib = G.load()
    names = declared_functions()
    assert len(names) >= 9
    for n in names:
        assert hasattr(lib, n), f"{n} declared in gdn.h but not exported"
    assert set(B.EXPORTS) <= set(names)


def test_version_and_status_strings():
    assert G.gdn_version() >= 100
    for st in (0, -1, -2, -3, -4):
        assert G.status_string(st)
    assert "unknown" in G.status_string(7)


A = 1 << 20          # a fake, 16-byte-aligned "device address": never dereferenced


def call_fwd(**kw):
    args = dict(q=A, k=2 * A, v=3 * A, gate=4 * A, beta=5 * A, state_in=None, state_out=None,
                out=6 * A, B=1, H=2, T=64, dk=32, dv=32, frame_len=16, chunk_len=16)
    args.update(kw)
    lib = G.load()
    return lib.gdn_forward(args["q"], args["k"], args["v"], args["gate"], args["beta"],
                           args["state_in"], args["state_out"], args["out"], args["B"], args["H"],
                           args["T"], args["dk"], args["dv"], args["frame_len"],
                           args["chunk_len"], None)


@pytest.mark.parametrize("kw,expect", [
    (dict(q=None), G.GDN_ERR_INVALID_ARG),
    (dict(k=None), G.GDN_ERR_INVALID_ARG),
    (dict(v=None), G.GDN_ERR_INVALID_ARG),
    (dict(gate=None), G.GDN_ERR_INVALID_ARG),
    (dict(beta=None), G.GDN_ERR_INVALID_ARG),
    (dict(out=None), G.GDN_ERR_INVALID_ARG),
    (dict(B=0), G.GDN_ERR_INVALID_ARG),
    (dict(H=0), G.GDN_ERR_INVALID_ARG),
    (dict(T=-1), G.GDN_ERR_INVALID_ARG),
    (dict(frame_len=0), G.GDN_ERR_INVALID_ARG),
    (dict(dk=0), G.GDN_ERR_INVALID_ARG),
    (dict(dk=24), G.GDN_ERR_UNSUPPORTED),
    (dict(dv=144), G.GDN_ERR_UNSUPPORTED),
    (dict(dk=8), G.GDN_ERR_UNSUPPORTED),
    (dict(chunk_len=128), G.GDN_ERR_UNSUPPORTED),
    (dict(chunk_len=48), G.GDN_ERR_UNSUPPORTED),
    (dict(q=A + 8), G.GDN_ERR_INVALID_ARG),            # misaligned
    (dict(out=6 * A + 2), G.GDN_ERR_INVALID_ARG),
    (dict(state_in=7 * A + 4), G.GDN_ERR_INVALID_ARG),
    (dict(gate=4 * A + 2), G.GDN_ERR_INVALID_ARG),
    (dict(out=A + 64), G.GDN_ERR_INVALID_ARG),         # out overlaps q
    (dict(out=5 * A), G.GDN_ERR_INVALID_ARG),          # out overlaps beta
    (dict(state_out=A), G.GDN_ERR_INVALID_ARG),        # state_out overlaps q
])
def test_forward_rejects_bad_arguments(kw, expect):
    assert call_fwd(**kw) == expect


def test_state_step_requires_state():
    lib = G.load()
    st = lib.gdn_state_step(A, 2 * A, 3 * A, 4 * A, 5 * A, None, 6 * A, 1, 2, 64, 32, 32, 16, 16, None)
    assert st == G.GDN_ERR_INVALID_ARG


def test_f32_entry_points_validate_too():
    lib = G.load()
    st = lib.gdn_forward_f32(A, 2 * A, 3 * A, 4 * A, 5 * A, None, None, 6 * A, 1, 2, 64, 32, 40,
                             16, 16, None)
    assert st == G.GDN_ERR_UNSUPPORTED
    st = lib.gdn_state_step_f32(A, 2 * A, 3 * A, 4 * A, 5 * A, None, None, 1, 2, 64, 32, 32,
                                16, 16, None)
    assert st == G.GDN_ERR_INVALID_ARG


def test_host_entry_validates_before_copying():
    lib = G.load()
    # missing host output buffer
    st = lib.gdn_forward_host(A, A, A, A, A, None, None, None, A, 2 * A, 3 * A, 4 * A, 5 * A,
                              None, 6 * A, 1, 2, 64, 32, 32, 16, 16, None)
    assert st == G.GDN_ERR_INVALID_ARG
    # a host state without a device state buffer
    st = lib.gdn_forward_host(A, A, A, A, A, A, None, A, A, 2 * A, 3 * A, 4 * A, 5 * A,
                              None, 6 * A, 1, 2, 64, 32, 32, 16, 16, None)
    assert st == G.GDN_ERR_INVALID_ARG


def test_binding_raises_on_error():
    with pytest.raises(G.GdnError) as e:
        G.gdn_forward(A, 2 * A, 3 * A, 4 * A, 5 * A, None, None, 6 * A, 1, 2, 64, 24, 32, 16, 16,
                      stream=0)
    assert e.value.status == G.GDN_ERR_UNSUPPORTED


def test_workspace_size_query_validates():
    import ctypes
    lib = G.load()
    n = ctypes.c_size_t(123)
    assert lib.gdn_workspace_bytes(1, 2, 64, 32, 32, 64, None) == G.GDN_ERR_INVALID_ARG
    assert lib.gdn_workspace_bytes(0, 2, 64, 112, 112, 64, ctypes.byref(n)) == G.GDN_ERR_INVALID_ARG
    assert lib.gdn_workspace_bytes(1, 2, 64, 24, 112, 64, ctypes.byref(n)) == G.GDN_ERR_UNSUPPORTED
    assert lib.gdn_workspace_bytes(1, 2, 64, 112, 112, 48, ctypes.byref(n)) == G.GDN_ERR_UNSUPPORTED
    # sizes served without a workspace answer 0 without touching the device
    for dims in ((1, 2, 64, 32, 32, 64), (1, 2, 64, 112, 112, 32), (1, 2, 0, 112, 112, 64),
                 (1, 2, 64, 64, 112, 64)):
        n.value = 123
        assert lib.gdn_workspace_bytes(*dims, ctypes.byref(n)) == G.GDN_OK
        assert n.value == 0


def test_workspace_entry_points_validate_first():
    lib = G.load()
    # argument errors come before any workspace or device check
    st = lib.gdn_forward_ws(None, 2 * A, 3 * A, 4 * A, 5 * A, None, None, 6 * A, 1, 2, 64, 112,
                            112, 16, 64, None, 0, None)
    assert st == G.GDN_ERR_INVALID_ARG
    st = lib.gdn_forward_ws(A, 2 * A, 3 * A, 4 * A, 5 * A, None, None, 6 * A, 1, 2, 64, 24,
                            112, 16, 64, None, 0, None)
    assert st == G.GDN_ERR_UNSUPPORTED
    st = lib.gdn_state_step_ws(A, 2 * A, 3 * A, 4 * A, 5 * A, None, 6 * A, 1, 2, 64, 112, 112,
                               16, 64, 7 * A, 1 << 20, None)
    assert st == G.GDN_ERR_INVALID_ARG      # no state
    # the host-buffer form refuses a missing workspace before copying anything
    st = lib.gdn_forward_host_ws(A, A, A, A, A, None, None, A, A, 2 * A, 3 * A, 4 * A, 5 * A,
                                 None, 6 * A, 1, 2, 64, 112, 112, 16, 64, None, 0, None)
    assert st == G.GDN_ERR_INVALID_ARG


def test_static_scratch_entry_validates_first():
    lib = G.load()
    st = lib.gdn_forward_static_ws(None, 2 * A, 3 * A, 4 * A, 5 * A, None, None, 6 * A, 1, 2, 64, 112, 112,
                                   16, 64, None)
    assert st == G.GDN_ERR_INVALID_ARG
    st = lib.gdn_forward_static_ws(A, 2 * A, 3 * A, 4 * A, 5 * A, None, None, 6 * A, 1, 2, 64, 40, 112,
                                   16, 64, None)
    assert st == G.GDN_ERR_UNSUPPORTED


def test_gated_entry_points_validate_gate_mode():
    lib = G.load()
    st = lib.gdn_forward_gated(A, 2 * A, 3 * A, 4 * A, 5 * A, None, None, 6 * A, 1, 2, 64, 32, 32, 16, 16,
                               2, None, 0, None)
    assert st == G.GDN_ERR_INVALID_ARG
    st = lib.gdn_forward_gated_f32(A, 2 * A, 3 * A, 4 * A, 5 * A, None, None, 6 * A, 1, 2, 64, 32, 32, 16, 16,
                                   -1, None)
    assert st == G.GDN_ERR_INVALID_ARG
    st = lib.gdn_forward_gated(None, 2 * A, 3 * A, 4 * A, 5 * A, None, None, 6 * A, 1, 2, 64, 32, 32, 16, 16,
                               1, None, 0, None)
    assert st == G.GDN_ERR_INVALID_ARG


def test_wait_limit_setter_needs_no_device():
    # sets a process-wide host value read at the next launch; 0 restores the default
    assert G.gdn_set_wait_limit_ns(1000) == G.GDN_OK
    assert G.gdn_set_wait_limit_ns(0) == G.GDN_OK


def test_bidirectional_entry_points_validate_before_any_device_work():
    lib = G.load()
    n = ctypes.c_size_t(7)
    assert lib.gdn_bidir_workspace_bytes(1, 2, 10, 64, 64, 64, 3, ctypes.byref(n)) == G.GDN_ERR_INVALID_ARG
    assert n.value == 0
    assert lib.gdn_bidir_workspace_bytes(1, 2, 10, 40, 64, 64, 2, ctypes.byref(n)) == G.GDN_ERR_UNSUPPORTED
    assert lib.gdn_bidir_workspace_bytes(1, 2, 0, 112, 112, 64, 2, ctypes.byref(n)) == G.GDN_OK
    assert n.value == 0
    # sizes without the ring need no device query: reversed q, k, v, gates, beta, backward output
    assert G.gdn_bidir_workspace_bytes(1, 2, 10, 64, 64, 64) == 3 * 2560 + 2 * 256 + 2560
    assert G.gdn_bidir_workspace_bytes(1, 2, 10, 64, 64, 64, 4) == 3 * 5120 + 2 * 256 + 5120
    # null input, no workspace, bad chunk: refused before any CUDA call
    st = lib.gdn_forward_bidir(None, 2 * A, 3 * A, 4 * A, 5 * A, 6 * A, 1, 2, 10, 64, 64, 4, 64, 7 * A, 1 << 20, None)
    assert st == G.GDN_ERR_INVALID_ARG
    st = lib.gdn_forward_bidir(A, 2 * A, 3 * A, 4 * A, 5 * A, 6 * A, 1, 2, 10, 64, 64, 4, 64, None, 0, None)
    assert st == G.GDN_ERR_INVALID_ARG
    st = lib.gdn_forward_bidir_f32(A, 2 * A, 3 * A, 4 * A, 5 * A, 6 * A, 1, 2, 10, 64, 64, 4, 48, 7 * A, 1 << 20,
                                   None)
    assert st == G.GDN_ERR_UNSUPPORTED
    # T = 0: nothing to do, nothing enqueued
    st = lib.gdn_forward_bidir(A, 2 * A, 3 * A, 4 * A, 5 * A, 6 * A, 1, 2, 0, 112, 112, 880, 64, None, 0, None)
    assert st == G.GDN_OK


def test_softmax_attention_validates_before_any_device_work():
    lib = G.load()
    args = (A, 2 * A, 3 * A, 5 * A)
    # unsupported head sizes, bad geometry, null or misaligned pointers, overlapping output
    assert lib.gdn_softmax_attention(*args, 1, 2, 64, 64, 64, 16, 3, 2, 1, None) == G.GDN_ERR_UNSUPPORTED
    assert lib.gdn_softmax_attention(*args, 1, 2, 64, 112, 72, 16, 3, 2, 1, None) == G.GDN_ERR_UNSUPPORTED
    assert lib.gdn_softmax_attention(*args, 1, 2, 64, 112, 112, 0, 3, 2, 1, None) == G.GDN_ERR_INVALID_ARG
    assert lib.gdn_softmax_attention(*args, 1, 2, 64, 112, 112, 16, 0, 2, 1, None) == G.GDN_ERR_INVALID_ARG
    assert lib.gdn_softmax_attention(*args, 1, 2, 64, 112, 112, 16, 3, -1, 1, None) == G.GDN_ERR_INVALID_ARG
    assert lib.gdn_softmax_attention(*args, 1, 2, 64, 112, 112, 16, 3, 2, -1, None) == G.GDN_ERR_INVALID_ARG
    assert lib.gdn_softmax_attention(*args, 0, 2, 64, 112, 112, 16, 3, 2, 1, None) == G.GDN_ERR_INVALID_ARG
    assert lib.gdn_softmax_attention(*args, 1, 70000, 64, 112, 112, 16, 3, 2, 1, None) == G.GDN_ERR_INVALID_ARG
    assert lib.gdn_softmax_attention(None, 2 * A, 3 * A, 5 * A, 1, 2, 64, 112, 112, 16, 3, 2, 1,
                                     None) == G.GDN_ERR_INVALID_ARG
    assert lib.gdn_softmax_attention(A + 8, 2 * A, 3 * A, 5 * A, 1, 2, 64, 112, 112, 16, 3, 2, 1,
                                     None) == G.GDN_ERR_INVALID_ARG
    assert lib.gdn_softmax_attention(A, 2 * A, 3 * A, A + 64, 1, 2, 64, 112, 112, 16, 3, 2, 1,
                                     None) == G.GDN_ERR_INVALID_ARG
    # T = 0: nothing to do, nothing enqueued
    assert lib.gdn_softmax_attention(*args, 1, 2, 0, 112, 112, 16, 3, 2, 1, None) == G.GDN_OK


def test_fp8_entry_validates_before_any_device_work():
    """gdn_forward_fp8 rejects a bad scale, unsupported sizes, null, misaligned or
    overlapping buffers on the host (fake device addresses, never dereferenced)."""
    lib = G.load()

    def call(q8=A, k8=2 * A, v8=3 * A, v_scale=0.5, out=6 * A, state_in=None, state_out=None,
             B=1, H=2, T=64, d=32, frame_len=16, chunk_len=64):
        return lib.gdn_forward_fp8(q8, k8, v8, v_scale, 4 * A, 5 * A, state_in, state_out, out,
                                   B, H, T, d, d, frame_len, chunk_len, None)

    for bad in (-1.0, float("nan"), float("inf"), -1e-30):
        assert call(v_scale=bad) == G.GDN_ERR_INVALID_ARG, bad
    assert call(d=128) == G.GDN_ERR_UNSUPPORTED            # above the e4m3 kernel's 112
    assert call(chunk_len=32) == G.GDN_ERR_UNSUPPORTED
    assert call(q8=None) == G.GDN_ERR_INVALID_ARG
    assert call(v8=None) == G.GDN_ERR_INVALID_ARG
    assert call(out=None) == G.GDN_ERR_INVALID_ARG
    assert call(k8=2 * A + 8) == G.GDN_ERR_INVALID_ARG    # not 16-byte aligned
    # out is bf16: 2 bytes per element against the inputs' 1, so it reaches v8 from below
    n = 1 * 64 * 2 * 32
    assert call(out=3 * A - n) == G.GDN_ERR_INVALID_ARG
    assert call(B=0) == G.GDN_ERR_INVALID_ARG
    assert call(frame_len=0) == G.GDN_ERR_INVALID_ARG
