"""GPU parity: the CUDA library against the float64 oracle on seeded inputs.

Bars: bf16 I/O -- max-abs <= 2e-2 and relative L2 <= 5e-3 on out and on the
final state; float32 reference mode -- relative L2 <= 1e-4.  Every call goes
through the C ABI (ctypes binding); outputs are NaN-filled and guarded.
"""

import numpy as np
import pytest

from oracle import gdn_reference as R
from workloads import (BLOCK, CLIP241, MINUTE, SESSIONS, TINY, draw, long_memory, make_inputs,
                       make_session_blocks)

from gpu_util import (assert_bf16_parity, assert_f32_parity, f32_device, host, run_library,
                      upload, rel_l2)

pytestmark = pytest.mark.gpu


def oracle(inp, state_in=None):
    Bn, T, H, dk = inp.q.shape
    if Bn * T * H <= 20000:
        return R.token_recurrence(inp, state_in)
    return R.c_forward(inp, state_in)


def check(inp, device, state_in=None, chunk_len=64, what=""):
    o, s = run_library(inp, device, state_in=state_in, chunk_len=chunk_len)
    ro, rs = oracle(inp, state_in)
    if inp.io_dtype == "f32":
        assert_f32_parity(o, ro, what + " out")
        assert_f32_parity(s, rs, what + " state")
    else:
        assert_bf16_parity(o, ro, what + " out")
        assert_bf16_parity(s, rs, what + " state")


# ---------------------------------------------------------------- small configs

@pytest.mark.parametrize("chunk_len", [16, 32, 64])
def test_tiny_f32_mode(cuda, chunk_len):
    inp = make_inputs(TINY)
    check(inp, cuda, chunk_len=chunk_len, what="tiny f32")


@pytest.mark.parametrize("chunk_len", [16, 32, 64])
def test_tiny_bf16(cuda, chunk_len):
    inp = make_inputs(TINY.with_(io_dtype="bf16"))
    check(inp, cuda, chunk_len=chunk_len, what="tiny bf16")


def test_block_bf16_state_in_out(cuda):
    inp = make_inputs(BLOCK)
    check(inp, cuda, state_in=inp.state, what="block")


def test_block_long_memory(cuda):
    inp = make_inputs(long_memory(BLOCK))
    check(inp, cuda, state_in=inp.state, what="block long-memory")


def test_block_f32_mode(cuda):
    inp = make_inputs(BLOCK.with_(io_dtype="f32", H=4))
    check(inp, cuda, state_in=inp.state, what="block f32")


def test_block_f32_mode_long_memory(cuda):
    inp = make_inputs(long_memory(BLOCK.with_(io_dtype="f32", H=4)))
    check(inp, cuda, state_in=inp.state, what="block f32 long-memory")


# ---------------------------------------------------------------- edge cases

EDGE = [
    # (B, H, T, dk, dv, frame_len, chunk_len, io, with_state)
    (1, 1, 1, 16, 16, 1, 64, "bf16", True),
    (1, 2, 17, 32, 32, 7, 16, "bf16", True),
    (2, 3, 63, 64, 64, 10, 64, "bf16", False),
    (1, 2, 65, 112, 112, 880, 64, "bf16", True),
    (1, 2, 130, 112, 112, 30, 32, "bf16", True),
    (2, 1, 200, 16, 128, 50, 64, "bf16", True),
    (1, 2, 150, 128, 16, 1, 64, "bf16", True),
    (1, 1, 300, 128, 128, 100, 64, "bf16", True),
    (1, 2, 129, 48, 80, 3, 16, "f32", True),
    (2, 2, 97, 112, 112, 880, 64, "f32", True),
]


@pytest.mark.parametrize("case", EDGE, ids=lambda c: "B{}H{}T{}dk{}dv{}f{}C{}{}{}".format(*c[:8], "s" if c[8] else ""))
def test_edge_shapes(cuda, case):
    Bn, H, T, dk, dv, fl, C, io, ws = case
    rng = np.random.Generator(np.random.PCG64(1234 + T))
    inp = draw(rng, Bn, H, T, dk, dv, fl, io, gate_mean=0.0, gate_std=1.5,
               state_std=0.3 if ws else None)
    check(inp, cuda, state_in=inp.state, chunk_len=C, what=str(case))


def test_empty_sequence_passes_state_through(cuda):
    import torch
    import hybrid_linear_attention_frame_b200 as G
    rng = np.random.Generator(np.random.PCG64(7))
    inp = draw(rng, 1, 2, 1, 32, 32, 4, "bf16", 0.0, 1.0, state_std=1.0)
    q, k, v, g, b = upload(inp, cuda)
    s_in = f32_device(inp.state, cuda)
    s_out = torch.full_like(s_in, float("nan"))
    out = torch.empty((1, 0, 2, 32), dtype=torch.bfloat16, device=cuda)
    G.gdn_forward(q, k, v, g, b, s_in, s_out, out if out.numel() else q.new_empty(8), 1, 2, 0,
                  32, 32, 4, 64)
    torch.cuda.synchronize()
    assert torch.equal(s_out, s_in)
    s_out.fill_(float("nan"))
    G.gdn_forward(q, k, v, g, b, None, s_out, q.new_empty(8), 1, 2, 0, 32, 32, 4, 64)
    torch.cuda.synchronize()
    assert bool((s_out == 0).all())


# ---------------------------------------------------------------- streaming

def test_state_step_composes(cuda):
    """One gdn_forward over two blocks == two in-place gdn_state_step calls."""
    import torch
    import hybrid_linear_attention_frame_b200 as G
    w = BLOCK.with_(H=4)
    inp = make_inputs(w, T=2 * w.T)
    Bn, T, H, dk = inp.q.shape
    o_full, s_full = run_library(inp, cuda, state_in=inp.state)
    q, k, v, g, b = upload(inp, cuda)
    state = f32_device(inp.state, cuda)
    T1 = w.T
    F1 = T1 // w.frame_len
    outs = []
    for (t0, t1, f0) in ((0, T1, 0), (T1, T, F1)):
        out = torch.empty((Bn, t1 - t0, H, 112), dtype=torch.bfloat16, device=cuda)
        G.gdn_state_step(q[:, t0:t1].contiguous(), k[:, t0:t1].contiguous(),
                         v[:, t0:t1].contiguous(), g[:, f0:].contiguous(),
                         b[:, t0:t1].contiguous(), state, out, Bn, H, t1 - t0, 112, 112,
                         w.frame_len, 64)
        outs.append(out)
    torch.cuda.synchronize()
    # chunk boundaries differ between the two schedules, so the results agree to
    # rounding (one bf16 ulp of the output), not bit for bit
    o_steps = host(torch.cat(outs, dim=1))
    assert_bf16_parity(o_steps, o_full, "two steps vs one call, out")
    assert_bf16_parity(host(state), s_full, "two steps vs one call, state")


def test_state_step_without_output_and_in_place_forward(cuda):
    import torch
    import hybrid_linear_attention_frame_b200 as G
    inp = make_inputs(BLOCK.with_(H=3))
    ro, rs = oracle(inp, inp.state)
    q, k, v, g, b = upload(inp, cuda)
    Bn, T, H, dk = inp.q.shape
    state = f32_device(inp.state, cuda)
    G.gdn_state_step(q, k, v, g, b, state, None, Bn, H, T, dk, dk, inp.frame_len, 64)
    torch.cuda.synchronize()
    assert_bf16_parity(host(state), rs, "commit-only state")
    state = f32_device(inp.state, cuda)
    out = torch.empty_like(v)
    G.gdn_forward(q, k, v, g, b, state, state, out, Bn, H, T, dk, dk, inp.frame_len, 64)
    torch.cuda.synchronize()
    assert_bf16_parity(host(state), rs, "in-place state")
    assert_bf16_parity(host(out), ro, "in-place out")


def test_host_buffer_entry_matches_device_entry(cuda):
    import torch
    import hybrid_linear_attention_frame_b200 as G
    inp = make_inputs(BLOCK.with_(H=2))
    o_dev, s_dev = run_library(inp, cuda, state_in=inp.state)
    q, k, v, g, b = (t.cpu().pin_memory() for t in upload(inp, cuda))
    Bn, T, H, dk = inp.q.shape
    h_state = torch.from_numpy(inp.state).pin_memory()
    h_state_out = torch.empty_like(h_state).pin_memory()
    h_out = torch.empty_like(v).pin_memory()
    d = [torch.empty_like(x, device=cuda) for x in (q, k, v, g, b)]
    d_state = torch.empty_like(h_state, device=cuda)
    d_out = torch.empty_like(v, device=cuda)
    G.gdn_forward_host(q, k, v, g, b, h_state, h_state_out, h_out, *d, d_state, d_out,
                       Bn, H, T, dk, dk, inp.frame_len, 64)
    np.testing.assert_array_equal(h_out.float().numpy(), o_dev.astype(np.float32))
    np.testing.assert_array_equal(h_state_out.numpy(), s_dev.astype(np.float32))


def test_host_buffer_entry_pipelined(cuda):
    """A clip-length layer (B 1, T 27,280) takes the segmented host path: copies of
    neighbouring segments overlap the computation, the state carried on the device.
    Against the oracle at the bf16 bars, and against the device entry (the same
    recurrence; the warm-up restarts differ, so rounding-level differences only)."""
    import torch
    import hybrid_linear_attention_frame_b200 as G
    w = CLIP241.with_(state_std=0.02)
    inp = make_inputs(w)
    o_dev, s_dev = run_library(inp, cuda, state_in=inp.state)
    q, k, v, g, b = (t.cpu().pin_memory() for t in upload(inp, cuda))
    Bn, T, H, dk = inp.q.shape
    h_state = torch.from_numpy(inp.state).pin_memory()
    h_state_out = torch.empty_like(h_state).pin_memory()
    h_out = torch.full_like(v, float("nan")).pin_memory()
    d = [torch.empty_like(x, device=cuda) for x in (q, k, v, g, b)]
    d_state = torch.empty_like(h_state, device=cuda)
    d_out = torch.empty_like(v, device=cuda)
    G.gdn_forward_host(q, k, v, g, b, h_state, h_state_out, h_out, *d, d_state, d_out,
                       Bn, H, T, dk, dk, inp.frame_len, 64)
    assert G.gdn_get_last_device_status() == G.GDN_OK
    o, s = h_out.float().numpy().astype(np.float64), h_state_out.numpy().astype(np.float64)
    assert not np.isnan(o).any()
    ro, rs = R.c_forward(inp, inp.state)
    assert_bf16_parity(o, ro, "pipelined host out")
    assert_bf16_parity(s, rs, "pipelined host state")
    assert rel_l2(o, o_dev) <= 1e-3 and rel_l2(s, s_dev) <= 1e-3


# ---------------------------------------------------------------- full sizes

def test_clip241_full(cuda):
    inp = make_inputs(CLIP241)
    check(inp, cuda, what="clip241")


@pytest.mark.slow
def test_minute_layer_full(cuda):
    """The benchmarked layer (T = 106,480, 20 heads) compared element by element."""
    inp = make_inputs(MINUTE)
    check(inp, cuda, what="minute")


def test_sessions_40_blocks_sampled(cuda):
    """4 sessions x 40 blocks through gdn_state_step with the state carried on the GPU;
    6 (session, head) chains are followed by the oracle over all 40 blocks."""
    import torch
    import hybrid_linear_attention_frame_b200 as G
    w = SESSIONS
    state0, blocks = make_session_blocks(w)
    state = f32_device(state0, cuda)
    picks = [(0, 0), (0, 19), (1, 7), (2, 3), (3, 11), (3, 19)]
    ss = [p[0] for p in picks]
    hh = [p[1] for p in picks]
    # the picked chains, stacked along B (H = 1), followed by the oracle in float64
    ref_state = state0[ss, hh][:, None].astype(np.float64)
    for n, blk in enumerate(blocks):
        q, k, v, g, b = upload(blk, cuda)
        out = torch.empty_like(v)
        G.gdn_state_step(q, k, v, g, b, state, out, w.B, w.H, w.T, w.d_k, w.d_v, w.frame_len, 64)
        torch.cuda.synchronize()
        o = host(out)[ss, :, hh][:, :, None]
        sub = type(blk)(q=blk.q[ss, :, hh][:, :, None], k=blk.k[ss, :, hh][:, :, None],
                        v=blk.v[ss, :, hh][:, :, None], gate=blk.gate[ss, :, hh][:, :, None],
                        beta=blk.beta[ss, :, hh][:, :, None], state=None,
                        io_dtype=blk.io_dtype, frame_len=blk.frame_len)
        ro, ref_state = R.c_forward(sub, ref_state)
        assert_bf16_parity(o, ro, f"block {n} out")
    sf = host(state)[ss, hh][:, None]
    assert_bf16_parity(sf, ref_state, "final state")
