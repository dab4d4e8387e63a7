"""GPU parity of the second gate placement (gate_mode 1: a frame's gate applied once,
at its first token) through gdn_forward_gated / gdn_forward_gated_f32, against the
float64 oracle run with the same placement.

Bars as everywhere: bf16 I/O -- max-abs <= 2e-2 and relative L2 <= 5e-3 on out and on
the final state; float32 reference mode -- relative L2 <= 1e-4.  Outputs are NaN-filled
before each call and must come back fully written.
"""

import dataclasses

import numpy as np
import pytest

from oracle import gdn_reference as R
from workloads import BLOCK, CLIP241, TINY, draw, long_memory, make_inputs

from gpu_util import assert_bf16_parity, assert_f32_parity, f32_device, host, upload

pytestmark = pytest.mark.gpu


def fs(inp):
    return dataclasses.replace(inp, gate_mode=R.GATE_FRAME_START)


def oracle(inp, state_in=None):
    Bn, T, H, dk = inp.q.shape
    if Bn * T * H <= 20000:
        return R.token_recurrence(inp, state_in)
    return R.c_forward(inp, state_in)


def run_gated(inp, device, state_in=None, chunk_len=64, ws=False, gate_mode=1):
    import torch
    import hybrid_linear_attention_frame_b200 as G
    q, k, v, g, b = upload(inp, device)
    Bn, T, H, dk = inp.q.shape
    dv = inp.v.shape[3]
    out = torch.full_like(v, float("nan"))
    st = torch.full((Bn, H, dk, dv), float("nan"), dtype=torch.float32, device=device)
    s_in = None if state_in is None else f32_device(state_in, device)
    if inp.io_dtype == "f32":
        G.gdn_forward_gated_f32(q, k, v, g, b, s_in, st, out, Bn, H, T, dk, dv, inp.frame_len, chunk_len,
                                gate_mode)
    else:
        wsp = G.workspace(Bn, H, T, dk, dv, chunk_len, device) if ws else None
        G.gdn_forward_gated(q, k, v, g, b, s_in, st, out, Bn, H, T, dk, dv, inp.frame_len, chunk_len,
                            gate_mode, wsp)
    torch.cuda.synchronize()
    assert G.gdn_get_last_device_status() == G.GDN_OK
    assert not bool(torch.isnan(out).any()) and not bool(torch.isnan(st).any()), "output not fully written"
    return host(out).reshape(Bn, T, H, dv), host(st).reshape(Bn, H, dk, dv)


def check(inp, device, state_in=None, chunk_len=64, ws=False, what=""):
    o, s = run_gated(inp, device, state_in, chunk_len, ws)
    ro, rs = oracle(inp, state_in)
    if inp.io_dtype == "f32":
        assert_f32_parity(o, ro, what + " out")
        assert_f32_parity(s, rs, what + " state")
    else:
        assert_bf16_parity(o, ro, what + " out")
        assert_bf16_parity(s, rs, what + " state")


@pytest.mark.parametrize("chunk_len", [16, 32, 64])
def test_tiny_f32_mode(cuda, chunk_len):
    check(fs(make_inputs(TINY)), cuda, chunk_len=chunk_len, what="tiny f32 frame-start")


@pytest.mark.parametrize("ws", [False, True], ids=["plain", "ring"])
def test_block_state_in_out(cuda, ws):
    inp = fs(make_inputs(BLOCK))
    check(inp, cuda, state_in=inp.state, ws=ws, what="block frame-start")


@pytest.mark.parametrize("ws", [False, True], ids=["plain", "ring"])
def test_block_long_memory(cuda, ws):
    inp = fs(make_inputs(long_memory(BLOCK)))
    check(inp, cuda, state_in=inp.state, ws=ws, what="block long-memory frame-start")


def test_block_f32_mode(cuda):
    inp = fs(make_inputs(BLOCK.with_(io_dtype="f32", H=4)))
    check(inp, cuda, state_in=inp.state, what="block f32 frame-start")


EDGE = [
    # (B, H, T, dk, dv, frame_len, chunk_len, io, ws)
    (1, 2, 65, 112, 112, 30, 64, "bf16", True),
    (2, 3, 200, 96, 80, 7, 64, "bf16", True),
    (1, 2, 333, 128, 128, 100, 64, "bf16", False),
    (1, 3, 150, 64, 64, 13, 64, "bf16", False),
    (2, 2, 97, 48, 32, 5, 32, "f32", False),
]


@pytest.mark.parametrize("case", EDGE, ids=lambda c: "B{}H{}T{}dk{}dv{}f{}C{}{}{}".format(*c[:8], "ws" if c[8] else ""))
def test_edge_shapes(cuda, case):
    Bn, H, T, dk, dv, fl, C, io, ws = case
    rng = np.random.Generator(np.random.PCG64(777 + T))
    inp = fs(draw(rng, Bn, H, T, dk, dv, fl, io, gate_mean=0.0, gate_std=1.5, state_std=0.3))
    check(inp, cuda, state_in=inp.state, chunk_len=C, ws=ws, what=str(case))


def test_clip241_ring(cuda):
    check(fs(make_inputs(CLIP241)), cuda, ws=True, what="clip241 frame-start")


def test_every_token_mode_equals_gdn_forward(cuda):
    """gate_mode 0 through the gated entry is gdn_forward itself, bit for bit."""
    import torch
    import hybrid_linear_attention_frame_b200 as G
    inp = make_inputs(BLOCK.with_(H=4))
    o0, s0 = run_gated(inp, cuda, inp.state, gate_mode=0)
    q, k, v, g, b = upload(inp, cuda)
    Bn, T, H, dk = inp.q.shape
    out = torch.empty_like(v)
    st = torch.empty((Bn, H, dk, dk), dtype=torch.float32, device=cuda)
    G.gdn_forward(q, k, v, g, b, f32_device(inp.state, cuda), st, out, Bn, H, T, dk, dk, inp.frame_len, 64)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(o0, host(out).reshape(o0.shape))
    np.testing.assert_array_equal(s0, host(st).reshape(s0.shape))


def test_streaming_split_at_a_frame_boundary(cuda):
    """Two gated calls (880 + 1760 tokens, the state carried) against one call."""
    inp = fs(make_inputs(BLOCK.with_(H=3)))
    o_full, s_full = run_gated(inp, cuda, inp.state, ws=True)
    t1 = inp.frame_len
    a = dataclasses.replace(inp, q=inp.q[:, :t1], k=inp.k[:, :t1], v=inp.v[:, :t1], gate=inp.gate[:, :1],
                            beta=inp.beta[:, :t1])
    b = dataclasses.replace(inp, q=inp.q[:, t1:], k=inp.k[:, t1:], v=inp.v[:, t1:], gate=inp.gate[:, 1:],
                            beta=inp.beta[:, t1:])
    oa, sa = run_gated(a, cuda, inp.state, ws=True)
    ob, sb = run_gated(b, cuda, sa.astype(np.float32), ws=True)
    assert_bf16_parity(np.concatenate([oa, ob], axis=1), o_full, "two calls vs one, out")
    assert_bf16_parity(sb, s_full, "two calls vs one, state")
