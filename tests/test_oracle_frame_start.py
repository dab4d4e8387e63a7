"""Pins of the oracle's second gate placement (gate_mode 1: a frame's gate applies
once, at the frame's first token; the other reading of "frame-wise" in the sglang
cookbook SANA-WM page, section 1 architecture table).  Every form of the oracle
(numpy token loop, chunked at C = 4 and 64, C recurrence, brute force) must pass
every pin.  CPU only.
"""

import dataclasses

import numpy as np
import pytest

from oracle import gdn_reference as R

from test_oracle_pins import BIG, IMPLS, mk, rand_inputs, read_golden


def fs(inp):
    return dataclasses.replace(inp, gate_mode=R.GATE_FRAME_START)


def pin_golden_pure_decay(fn):
    g = read_golden("worked_example_frame_start.txt")
    T = len(g["out"])
    inp = fs(mk(np.ones((1, T, 1, 1)), np.ones((1, T, 1, 1)), np.zeros((1, T, 1, 1)),
                np.reshape(g["gate"], (1, -1, 1)), -BIG * np.ones((1, T, 1)),
                frame_len=int(g["frame_len"][0])))
    out, S = fn(inp, np.reshape(g["state_in"], (1, 1, 1, 1)), eps=0.0)
    # the logits +-ln 3 reach the method as float32 (relative error 3e-8 in g)
    np.testing.assert_allclose(out.ravel(), g["out"], rtol=2e-7, atol=0)


def pin_golden_writes(fn):
    g = read_golden("worked_example_frame_start_writes.txt")
    T = len(g["out"])
    inp = fs(mk(np.ones((1, T, 1, 1)), np.ones((1, T, 1, 1)), np.reshape(g["v"], (1, T, 1, 1)),
                np.reshape(g["gate"], (1, -1, 1)), np.reshape(g["beta"], (1, T, 1)),
                frame_len=int(g["frame_len"][0])))
    out, S = fn(inp, np.reshape(g["state_in"], (1, 1, 1, 1)), eps=0.0)
    np.testing.assert_allclose(out.ravel(), g["out"], rtol=2e-7, atol=0)
    np.testing.assert_allclose(S.ravel(), g["state_out"], rtol=2e-7, atol=0)


def pin_pure_decay_closed_form(fn):
    """beta = 0: S_t = prod over the frames started by t of 1/(1 + e^{g_f}) S0."""
    inp = fs(rand_inputs(3, T=11, frame_len=3))
    inp.beta[:] = -BIG
    out, S = fn(inp, inp.state, eps=0.0)
    g = inp.gate.astype(np.float64)
    S0 = inp.state.astype(np.float64)
    qn = inp.q.astype(np.float64) / np.linalg.norm(inp.q.astype(np.float64), axis=-1, keepdims=True)
    T = inp.q.shape[1]
    for t in range(T):
        frames = t // 3 + 1                            # frames 0 .. f(t) have started
        decay = np.prod(1.0 / (1.0 + np.exp(g[:, :frames, :])), axis=1)     # [B, H]
        expect = np.einsum("bhij,bhi->bhj", decay[:, :, None, None] * S0, qn[:, t])
        np.testing.assert_allclose(out[:, t], expect, rtol=1e-12, atol=1e-13)


def pin_one_frame_is_ungated_rule(fn):
    """Inside one frame only its first token decays: a call that stays inside frame 0
    equals the ungated rule (a = 1) started from a_0 S0 (the every-token form with
    gate logits at -1e4, pinned independently)."""
    inp = fs(rand_inputs(4, T=7, frame_len=7))
    out, S = fn(inp, inp.state, eps=0.0)
    a0 = 1.0 / (1.0 + np.exp(inp.gate[:, 0, :].astype(np.float64)))          # [B, H]
    ref = dataclasses.replace(inp, gate=np.full_like(inp.gate, -BIG), gate_mode=R.GATE_EVERY_TOKEN)
    o2, S2 = fn(ref, a0[:, :, None, None] * inp.state.astype(np.float64), eps=0.0)
    np.testing.assert_allclose(out, o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(S, S2, rtol=0, atol=1e-12)


def pin_frame_len_one_equals_every_token(fn):
    """With one token per frame both placements are the same rule."""
    inp = rand_inputs(5, T=9, frame_len=1)
    o0, S0 = fn(inp, inp.state)
    o1, S1 = fn(fs(inp), inp.state)
    np.testing.assert_allclose(o1, o0, rtol=0, atol=1e-13)
    np.testing.assert_allclose(S1, S0, rtol=0, atol=1e-13)


def pin_streaming_composition(fn):
    """Two calls split at a frame boundary, the state carried, equal one call."""
    inp = fs(rand_inputs(6, T=12, frame_len=4))
    o, S = fn(inp, inp.state)
    t1 = 8
    a = dataclasses.replace(inp, q=inp.q[:, :t1], k=inp.k[:, :t1], v=inp.v[:, :t1],
                            gate=inp.gate[:, :2], beta=inp.beta[:, :t1])
    b = dataclasses.replace(inp, q=inp.q[:, t1:], k=inp.k[:, t1:], v=inp.v[:, t1:],
                            gate=inp.gate[:, 2:], beta=inp.beta[:, t1:])
    oa, Sa = fn(a, inp.state)
    ob, Sb = fn(b, Sa)
    np.testing.assert_allclose(np.concatenate([oa, ob], axis=1), o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(Sb, S, rtol=0, atol=1e-12)


def pin_gate_reaches_only_frame_starts(fn):
    """Changing the gate of frame 1 changes nothing before frame 1 starts, and (with
    beta = 0 after it) scales the state from that token on by the ratio of the gates."""
    inp = fs(rand_inputs(7, T=10, frame_len=5))
    inp.beta[:, 5:] = -BIG
    o, S = fn(inp, inp.state)
    mod = dataclasses.replace(inp, gate=inp.gate.copy())
    mod.gate[:, 1, :] += 1.5
    o2, S2 = fn(mod, inp.state)
    np.testing.assert_allclose(o2[:, :5], o[:, :5], rtol=0, atol=0)
    ratio = (1.0 + np.exp(inp.gate[:, 1, :].astype(np.float64))) / (1.0 + np.exp(mod.gate[:, 1, :].astype(np.float64)))
    np.testing.assert_allclose(S2, ratio[:, :, None, None] * S, rtol=1e-10, atol=1e-14)


PINS = [pin_golden_pure_decay, pin_golden_writes, pin_pure_decay_closed_form,
        pin_one_frame_is_ungated_rule, pin_frame_len_one_equals_every_token,
        pin_streaming_composition, pin_gate_reaches_only_frame_starts]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
@pytest.mark.parametrize("impl", list(IMPLS), ids=str)
def test_frame_start_pin(impl, pin):
    pin(IMPLS[impl])


@pytest.mark.parametrize("C", [4, 16, 64])
@pytest.mark.parametrize("T", [1, 63, 130])
def test_chunked_equals_token_frame_start(C, T):
    inp = fs(rand_inputs(40 + T, B=2, H=3, T=T, dk=16, dv=8, frame_len=7, gate_mean=-1.0, gate_std=1.0))
    o1, S1 = R.token_recurrence(inp, inp.state)
    o2, S2 = R.chunked(inp, inp.state, chunk_len=C)
    scale = max(1.0, np.abs(o1).max())
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-11 * scale)
    np.testing.assert_allclose(S2, S1, rtol=0, atol=1e-11 * scale)


def test_modes_differ_when_frames_are_longer_than_one_token():
    inp = rand_inputs(8, T=12, frame_len=4)
    o0, _ = R.token_recurrence(inp, inp.state)
    o1, _ = R.token_recurrence(fs(inp), inp.state)
    assert np.abs(o1 - o0).max() > 1e-3


def test_unknown_gate_mode_is_refused():
    inp = dataclasses.replace(rand_inputs(9), gate_mode=2)
    with pytest.raises(ValueError):
        R.token_recurrence(inp)
