"""Pins of the oracle's bidirectional form: the forward scan plus the same rule run
from the last token to the first, both from a zero state, every token keeping its
own frame's gate (the reading of the dense checkpoint's "bidirectional" GDN, sglang
cookbook SANA-WM page, dense-bidirectional section, which the pages do not define).
Both forms (numpy and C) must pass every pin; the numpy backward loop alone is
pinned by the hand-derived examples too.  A mistake planted in a copy of the
backward loop must fail at least one pin.  CPU only.
"""

import dataclasses

import numpy as np
import pytest

from oracle import gdn_reference as R

from test_oracle_pins import BIG, mk, rand_inputs, read_golden


def impl_numpy(inp, eps=R.EPS):
    return R.bidirectional(inp, eps)


def impl_c(inp, eps=R.EPS):
    return R.c_bidirectional(inp, eps)


IMPLS = {"numpy": impl_numpy, "c": impl_c}


def forward(inp, eps=R.EPS):
    return R.token_recurrence(inp, None, eps)[0]


def reverse_tokens(inp):
    """The same sequence in reverse token order, frame by frame (T a multiple of frame_len)."""
    T, fl = inp.q.shape[1], inp.frame_len
    assert T % fl == 0
    return dataclasses.replace(inp, q=inp.q[:, ::-1].copy(), k=inp.k[:, ::-1].copy(), v=inp.v[:, ::-1].copy(),
                               beta=inp.beta[:, ::-1].copy(), gate=inp.gate[:, ::-1].copy(), state=None)


# ----------------------------------------------------------------------------
# pins
# ----------------------------------------------------------------------------

def golden_frames_inputs():
    g = read_golden("worked_example_bidirectional_frames.txt")
    T = len(g["out"])
    inp = mk(np.ones((1, T, 1, 1)), np.ones((1, T, 1, 1)), np.reshape(g["v"], (1, T, 1, 1)),
             np.reshape(g["gate"], (1, -1, 1)), np.reshape(g["beta"], (1, T, 1)),
             frame_len=int(g["frame_len"][0]))
    return inp, g


def golden_erase_inputs():
    g = read_golden("worked_example_bidirectional_erase.txt")
    inp = mk(np.reshape(g["q"], (1, 2, 1, 2)), np.reshape(g["k"], (1, 2, 1, 2)),
             np.reshape(g["v"], (1, 2, 1, 2)), -BIG * np.ones((1, 2, 1)), BIG * np.ones((1, 2, 1)),
             frame_len=1)
    return inp, g


def pin_golden_frames(fn):
    inp, g = golden_frames_inputs()
    # the logit ln 3 reaches the method as float32 (relative error 3e-8 in g)
    np.testing.assert_allclose(fn(inp, eps=0.0).ravel(), g["out"], rtol=2e-7, atol=0)


def pin_golden_erase(fn):
    inp, g = golden_erase_inputs()
    np.testing.assert_allclose(fn(inp, eps=0.0).ravel(), g["out"], rtol=0, atol=1e-12)


def pin_single_token(fn):
    """T = 1 from zero states: each scan gives b (q^ . k^) v, so o = 2 b (q^ . k^) v."""
    inp = rand_inputs(11, T=1, frame_len=1)
    out = fn(inp, eps=0.0)
    q = inp.q.astype(np.float64)
    k = inp.k.astype(np.float64)
    qk = np.sum(q * k, axis=-1) / (np.linalg.norm(q, axis=-1) * np.linalg.norm(k, axis=-1))     # [B,1,H]
    b = 1.0 / (1.0 + np.exp(-inp.beta.astype(np.float64)))
    expect = 2.0 * (b * qk)[..., None] * inp.v.astype(np.float64)
    np.testing.assert_allclose(out, expect, rtol=1e-12, atol=1e-14)


def pin_time_reversal(fn):
    """Reversing the tokens (and the frames with them) reverses the output."""
    inp = rand_inputs(12, B=2, H=2, T=12, frame_len=3)
    out = fn(inp)
    out_r = fn(reverse_tokens(inp))
    np.testing.assert_allclose(out_r[:, ::-1], out, rtol=0, atol=1e-12)


def pin_backward_half_is_anticausal(fn):
    """out - forward (the forward scan is pinned on its own) at token t depends on
    tokens t.. T-1 only: changing token s leaves it unchanged at t > s."""
    inp = rand_inputs(13, T=10, frame_len=2)
    base = fn(inp) - forward(inp)
    s = 6
    pert = dataclasses.replace(inp, q=inp.q.copy(), k=inp.k.copy(), v=inp.v.copy(), beta=inp.beta.copy())
    pert.k[:, s] += 0.7
    pert.v[:, s] -= 1.3
    pert.beta[:, s] += 0.9
    other = fn(pert) - forward(pert)
    np.testing.assert_allclose(other[:, s + 1:], base[:, s + 1:], rtol=0, atol=1e-12)
    assert np.max(np.abs(other[:, : s + 1] - base[:, : s + 1])) > 1e-3


def pin_backward_is_forward_of_reversed(fn):
    """The backward half equals the forward scan (pinned on its own) of the reversed
    sequence with each token's own gate, given one token per frame."""
    inp = rand_inputs(14, B=1, H=3, T=9, frame_len=3)
    T = inp.q.shape[1]
    tok_gate = inp.gate[:, np.arange(T) // inp.frame_len, :]           # [B, T, H]
    rev = dataclasses.replace(inp, q=inp.q[:, ::-1].copy(), k=inp.k[:, ::-1].copy(), v=inp.v[:, ::-1].copy(),
                              beta=inp.beta[:, ::-1].copy(), gate=tok_gate[:, ::-1].copy(), frame_len=1,
                              state=None)
    back = fn(inp) - forward(inp)
    np.testing.assert_allclose(back, forward(rev)[:, ::-1], rtol=0, atol=1e-12)


PINS = [pin_golden_frames, pin_golden_erase, pin_single_token, pin_time_reversal,
        pin_backward_half_is_anticausal, pin_backward_is_forward_of_reversed]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
@pytest.mark.parametrize("impl", sorted(IMPLS))
def test_bidirectional_pin(impl, pin):
    pin(IMPLS[impl])


def test_backward_loop_matches_hand_examples():
    inp, g = golden_frames_inputs()
    np.testing.assert_allclose(R.token_recurrence_backward(inp, eps=0.0).ravel(), g["backward"], rtol=2e-7)
    inp, g = golden_erase_inputs()
    np.testing.assert_allclose(R.token_recurrence_backward(inp, eps=0.0).ravel(), g["backward"], atol=1e-12)


@pytest.mark.parametrize("T,fl", [(0, 1), (1, 1), (7, 3), (20, 4)])
def test_numpy_and_c_forms_agree(T, fl):
    inp = rand_inputs(15, B=2, H=2, T=T, frame_len=fl)
    np.testing.assert_allclose(impl_c(inp), impl_numpy(inp), rtol=0, atol=1e-12)


def test_frame_start_placement_is_refused():
    inp = dataclasses.replace(rand_inputs(16), gate_mode=R.GATE_FRAME_START)
    with pytest.raises(ValueError):
        R.bidirectional(inp)
    with pytest.raises(ValueError):
        R.c_bidirectional(inp)


# ----------------------------------------------------------------------------
# planted mistakes: a copy of the backward loop with one error must fail a pin
# ----------------------------------------------------------------------------

def _mutant(kind):
    def backward(inp, eps):
        qn, kn, v, la, bt = R._prep(inp, eps)
        B, T, H, dk = qn.shape
        Rs = np.zeros((B, H, dk, v.shape[3]))
        out = np.zeros(v.shape)
        fl = inp.frame_len
        for t in range(T - 1, -1, -1):
            lt = la[:, T - 1 - t, :] if kind == "gate_of_mirrored_token" else la[:, t, :]
            if kind == "gate_of_mirrored_frame":
                F = inp.gate.shape[1]
                lt = -R.softplus(inp.gate[:, F - 1 - t // fl, :].astype(np.float64))
            a = np.exp(lt)[:, :, None, None]
            b = bt[:, t, :][:, :, None, None]
            k_t = kn[:, t]
            if kind == "output_before_update":
                out[:, t] = np.einsum("bhij,bhi->bhj", Rs, qn[:, t])
            kR = np.einsum("bhi,bhij->bhj", k_t, Rs)
            erase = 0.0 if kind == "no_erase" else b * k_t[..., :, None] * kR[..., None, :]
            Rs = a * (Rs - erase) + b * k_t[..., :, None] * v[:, t][..., None, :]
            if kind != "output_before_update":
                out[:, t] = np.einsum("bhij,bhi->bhj", Rs, qn[:, t])
        if kind == "forward_twice":
            return forward(inp, eps)
        return out

    def bidir(inp, eps=R.EPS):
        return forward(inp, eps) + backward(inp, eps)
    return bidir


@pytest.mark.parametrize("kind", ["gate_of_mirrored_token", "gate_of_mirrored_frame", "output_before_update",
                                  "no_erase", "forward_twice"])
def test_planted_mistake_fails_a_pin(kind):
    fn = _mutant(kind)
    failed = []
    for pin in PINS:
        try:
            pin(fn)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"mistake {kind} passes every pin"
