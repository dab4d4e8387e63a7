"""GPU parity with slowly decaying gates, where the carried state matters.

With the configs' gate logits ~ N(2, 0.5) a token's gate is about 0.12 and the
state forgets within a few dozen tokens, so the long-range carry (and the bf16
copy of the state that feeds the tensor cores) is hardly exercised.  Here the
gate logits are ~ N(-6, 0.5) (a ~ 0.9975, about 11 % of the state survives a
frame) and the state is carried across whole clips and across the 40 streaming
blocks of the batched-sessions workload, through every entry point that carries
it: gdn_forward and gdn_state_step (sequence-parallel kernel, whose stretches
then start from long warm-ups), gdn_forward_ws and gdn_state_step_ws (ring
kernel), and gdn_forward_gated (the frame-start gate placement).

Bars as everywhere for bf16 I/O: max-abs <= 2e-2 and relative L2 <= 5e-3 on out
and on the final state, against the float64 oracle.
"""

import numpy as np
import pytest

from oracle import gdn_reference as R
from workloads import CLIP241, MINUTE, SESSIONS, long_memory, make_inputs, make_session_blocks

from gpu_util import assert_bf16_parity, f32_device, host, run_library, upload

pytestmark = pytest.mark.gpu


def sessions_40_blocks(cuda, w, ws):
    """4 sessions x 40 blocks with the state carried on the GPU; 6 (session, head)
    chains followed by the oracle over all 40 blocks, every block's output compared."""
    import torch
    import hybrid_linear_attention_frame_b200 as G
    state0, blocks = make_session_blocks(w)
    state = f32_device(state0, cuda)
    wsp = G.workspace(w.B, w.H, w.T, w.d_k, w.d_v, 64, cuda) if ws else None
    picks = [(0, 0), (0, 19), (1, 7), (2, 3), (3, 11), (3, 19)]
    ss = [p[0] for p in picks]
    hh = [p[1] for p in picks]
    ref_state = state0[ss, hh][:, None].astype(np.float64)
    worst = 0.0
    for n, blk in enumerate(blocks):
        q, k, v, g, b = upload(blk, cuda)
        out = torch.empty_like(v)
        if ws:
            G.gdn_state_step_ws(q, k, v, g, b, state, out, w.B, w.H, w.T, w.d_k, w.d_v, w.frame_len, 64, wsp)
        else:
            G.gdn_state_step(q, k, v, g, b, state, out, w.B, w.H, w.T, w.d_k, w.d_v, w.frame_len, 64)
        torch.cuda.synchronize()
        assert G.gdn_get_last_device_status() == G.GDN_OK
        o = host(out)[ss, :, hh][:, :, None]
        sub = type(blk)(q=blk.q[ss, :, hh][:, :, None], k=blk.k[ss, :, hh][:, :, None],
                        v=blk.v[ss, :, hh][:, :, None], gate=blk.gate[ss, :, hh][:, :, None],
                        beta=blk.beta[ss, :, hh][:, :, None], state=None,
                        io_dtype=blk.io_dtype, frame_len=blk.frame_len)
        ro, ref_state = R.c_forward(sub, ref_state)
        worst = max(worst, assert_bf16_parity(o, ro, f"block {n} out")[1])
    sf = host(state)[ss, hh][:, None]
    assert_bf16_parity(sf, ref_state, "final state")
    return worst


@pytest.mark.parametrize("ws", [False, True], ids=["state_step", "state_step_ws"])
def test_sessions_40_blocks_long_memory(cuda, ws):
    sessions_40_blocks(cuda, long_memory(SESSIONS), ws)


def _full(cuda, w, ws, gate_mode=None):
    inp = make_inputs(w)
    if gate_mode is not None:
        inp.gate_mode = gate_mode
        o, s = run_gated(inp, cuda, ws)
    else:
        o, s = run_library(inp, cuda, state_in=None, ws=ws)
    ro, rs = R.c_forward(inp, None)
    assert_bf16_parity(o, ro, w.name + " out")
    assert_bf16_parity(s, rs, w.name + " state")


def run_gated(inp, cuda, ws):
    import torch
    import hybrid_linear_attention_frame_b200 as G
    q, k, v, g, b = upload(inp, cuda)
    Bn, T, H, dk = inp.q.shape
    dv = inp.v.shape[3]
    out = torch.full_like(v, float("nan"))
    st = torch.full((Bn, H, dk, dv), float("nan"), dtype=torch.float32, device=cuda)
    wsp = G.workspace(Bn, H, T, dk, dv, 64, cuda) if ws else None
    G.gdn_forward_gated(q, k, v, g, b, None, st, out, Bn, H, T, dk, dv, inp.frame_len, 64, inp.gate_mode, wsp)
    torch.cuda.synchronize()
    assert G.gdn_get_last_device_status() == G.GDN_OK
    assert not bool(torch.isnan(out).any()) and not bool(torch.isnan(st).any())
    return host(out).reshape(Bn, T, H, dv), host(st).reshape(Bn, H, dk, dv)


@pytest.mark.parametrize("ws", [False, True], ids=["forward", "forward_ws"])
def test_clip241_long_memory(cuda, ws):
    _full(cuda, long_memory(CLIP241), ws)


@pytest.mark.parametrize("ws", [False, True], ids=["gated", "gated_ws"])
def test_clip241_frame_start_placement(cuda, ws):
    """Frame-start placement (gate_mode 1) at clip length: one decay per frame, so the
    state is carried through whole frames undecayed."""
    _full(cuda, CLIP241, ws, gate_mode=1)


@pytest.mark.slow
def test_minute_layer_long_memory(cuda):
    """The benchmarked layer with slow gates: every stretch of the sequence-parallel
    kernel starts from a warm-up of about 200 chunks, or from the chain's start."""
    _full(cuda, long_memory(MINUTE), False)
