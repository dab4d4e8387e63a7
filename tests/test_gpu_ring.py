"""GPU parity of the workspace entry points (gdn_forward_ws, gdn_state_step_ws,
gdn_forward_host_ws): the shared-prep ring kernel against the float64 oracle.

Bars as for gdn_forward: bf16 I/O -- max-abs <= 2e-2 and relative L2 <= 5e-3 on
out and on the final state.  Outputs are NaN-filled and guarded; workspaces are
filled with garbage before every call.
"""

import numpy as np
import pytest

from oracle import gdn_reference as R
from workloads import BLOCK, CLIP241, MINUTE, SESSIONS, draw, long_memory, make_inputs, make_session_blocks

from gpu_util import assert_bf16_parity, f32_device, host, run_library, upload

pytestmark = pytest.mark.gpu


def oracle(inp, state_in=None):
    Bn, T, H, dk = inp.q.shape
    if Bn * T * H <= 20000:
        return R.token_recurrence(inp, state_in)
    return R.c_forward(inp, state_in)


def check(inp, device, state_in=None, what=""):
    o, s = run_library(inp, device, state_in=state_in, ws=True)
    ro, rs = oracle(inp, state_in)
    assert_bf16_parity(o, ro, what + " out")
    assert_bf16_parity(s, rs, what + " state")
    return o, s


def test_ring_path_needs_a_workspace(cuda):
    import hybrid_linear_attention_frame_b200 as G
    assert G.gdn_workspace_bytes(1, 20, 2640, 112, 112, 64) > 0
    # sizes that take a path without workspace report 0
    assert G.gdn_workspace_bytes(1, 20, 2640, 64, 64, 64) == 0
    assert G.gdn_workspace_bytes(1, 20, 2640, 112, 112, 32) == 0
    assert G.gdn_workspace_bytes(1, 20, 0, 112, 112, 64) == 0


def test_block_state_in_out(cuda):
    inp = make_inputs(BLOCK)
    check(inp, cuda, state_in=inp.state, what="block ws")


def test_block_long_memory(cuda):
    inp = make_inputs(long_memory(BLOCK))
    check(inp, cuda, state_in=inp.state, what="block long-memory ws")


def test_matches_plain_path(cuda):
    """Same kernels' arithmetic in the same order: the two paths agree to rounding."""
    inp = make_inputs(BLOCK.with_(H=6))
    o1, s1 = run_library(inp, cuda, state_in=inp.state)
    o2, s2 = run_library(inp, cuda, state_in=inp.state, ws=True)
    assert_bf16_parity(o2, o1, "ws vs plain out")
    assert_bf16_parity(s2, s1, "ws vs plain state")


RING_EDGE = [
    # (B, H, T, dk, dv, frame_len, with_state): d_k, d_v > 64 and chunk 64 take the ring
    (1, 1, 1, 112, 112, 1, True),
    (1, 2, 65, 112, 112, 880, True),
    (1, 3, 130, 80, 96, 30, True),
    (2, 1, 200, 128, 128, 50, False),
    (1, 2, 333, 96, 128, 7, True),
    (3, 5, 129, 112, 80, 64, True),
]


@pytest.mark.parametrize("case", RING_EDGE, ids=lambda c: "B{}H{}T{}dk{}dv{}f{}{}".format(*c[:6], "s" if c[6] else ""))
def test_edge_shapes(cuda, case):
    Bn, H, T, dk, dv, fl, ws = case
    rng = np.random.Generator(np.random.PCG64(4321 + T))
    inp = draw(rng, Bn, H, T, dk, dv, fl, "bf16", gate_mean=0.0, gate_std=1.5,
               state_std=0.3 if ws else None)
    check(inp, cuda, state_in=inp.state, what=str(case))


def test_more_chains_than_groups(cuda):
    """B*H = 160 chains: every group of CTAs serves several chains back to back."""
    rng = np.random.Generator(np.random.PCG64(99))
    inp = draw(rng, 8, 20, 150, 112, 112, 40, "bf16", gate_mean=-1.0, gate_std=1.0, state_std=0.2)
    check(inp, cuda, state_in=inp.state, what="160 chains")


def test_clip241_full(cuda):
    inp = make_inputs(CLIP241)
    check(inp, cuda, what="clip241 ws")


@pytest.mark.slow
def test_minute_layer_full(cuda):
    inp = make_inputs(MINUTE)
    check(inp, cuda, what="minute ws")


def test_state_step_ws_commit_only_and_in_place(cuda):
    import torch
    import hybrid_linear_attention_frame_b200 as G
    inp = make_inputs(BLOCK.with_(H=3))
    ro, rs = oracle(inp, inp.state)
    q, k, v, g, b = upload(inp, cuda)
    Bn, T, H, dk = inp.q.shape
    wsp = G.workspace(Bn, H, T, dk, dk, 64, cuda)
    state = f32_device(inp.state, cuda)
    G.gdn_state_step_ws(q, k, v, g, b, state, None, Bn, H, T, dk, dk, inp.frame_len, 64, wsp)
    torch.cuda.synchronize()
    assert_bf16_parity(host(state), rs, "commit-only state")
    state = f32_device(inp.state, cuda)
    out = torch.empty_like(v)
    G.gdn_forward_ws(q, k, v, g, b, state, state, out, Bn, H, T, dk, dk, inp.frame_len, 64, wsp)
    torch.cuda.synchronize()
    assert_bf16_parity(host(state), rs, "in-place state")
    assert_bf16_parity(host(out), ro, "in-place out")
    assert G.gdn_get_last_device_status() == G.GDN_OK


def test_workspace_checks(cuda):
    import torch
    import hybrid_linear_attention_frame_b200 as G
    inp = make_inputs(BLOCK.with_(H=2))
    q, k, v, g, b = upload(inp, cuda)
    Bn, T, H, dk = inp.q.shape
    out = torch.empty_like(v)
    n = G.gdn_workspace_bytes(Bn, H, T, dk, dk, 64)
    wsp = torch.empty(n + 512, dtype=torch.uint8, device=cuda)
    args = (q, k, v, g, b, None, None, out, Bn, H, T, dk, dk, inp.frame_len, 64)
    assert G.gdn_forward_ws(*args, None, 0, check=False) == G.GDN_ERR_INVALID_ARG
    assert G.gdn_forward_ws(*args, wsp, n - 16, check=False) == G.GDN_ERR_INVALID_ARG
    assert G.gdn_forward_ws(*args, wsp[16:], n, check=False) == G.GDN_ERR_INVALID_ARG   # misaligned
    assert G.gdn_forward_ws(*args, out, n, check=False) == G.GDN_ERR_INVALID_ARG       # overlaps out
    assert G.gdn_forward_ws(*args, wsp, n, check=False) == G.GDN_OK
    torch.cuda.synchronize()


def test_host_ws_entry_matches_device_ws_entry(cuda):
    import torch
    import hybrid_linear_attention_frame_b200 as G
    inp = make_inputs(BLOCK.with_(H=2))
    o_dev, s_dev = run_library(inp, cuda, state_in=inp.state, ws=True)
    q, k, v, g, b = (t.cpu().pin_memory() for t in upload(inp, cuda))
    Bn, T, H, dk = inp.q.shape
    h_state = torch.from_numpy(inp.state).pin_memory()
    h_state_out = torch.empty_like(h_state).pin_memory()
    h_out = torch.empty_like(v).pin_memory()
    d = [torch.empty_like(x, device=cuda) for x in (q, k, v, g, b)]
    d_state = torch.empty_like(h_state, device=cuda)
    d_out = torch.empty_like(v, device=cuda)
    wsp = G.workspace(Bn, H, T, dk, dk, 64, cuda)
    G.gdn_forward_host_ws(q, k, v, g, b, h_state, h_state_out, h_out, *d, d_state, d_out,
                          Bn, H, T, dk, dk, inp.frame_len, 64, wsp)
    np.testing.assert_array_equal(h_out.float().numpy(), o_dev.astype(np.float32))
    np.testing.assert_array_equal(h_state_out.numpy(), s_dev.astype(np.float32))


def test_sessions_40_blocks_sampled(cuda):
    """4 sessions x 40 blocks through gdn_state_step_ws (80 chains per call)."""
    import torch
    import hybrid_linear_attention_frame_b200 as G
    w = SESSIONS
    state0, blocks = make_session_blocks(w)
    state = f32_device(state0, cuda)
    wsp = G.workspace(w.B, w.H, w.T, w.d_k, w.d_v, 64, cuda)
    picks = [(0, 0), (1, 19), (2, 3), (3, 11)]
    ss = [p[0] for p in picks]
    hh = [p[1] for p in picks]
    ref_state = state0[ss, hh][:, None].astype(np.float64)
    for n, blk in enumerate(blocks):
        q, k, v, g, b = upload(blk, cuda)
        out = torch.empty_like(v)
        G.gdn_state_step_ws(q, k, v, g, b, state, out, w.B, w.H, w.T, w.d_k, w.d_v, w.frame_len, 64, wsp)
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
