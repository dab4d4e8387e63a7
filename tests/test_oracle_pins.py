"""Pins for the float64 oracle: each check comes from the mathematics of the
gated delta rule, not from the oracle's own code.

* two worked examples derived by hand (tests/golden/, exact rationals);
* closed forms: identity (a = 1, beta = 0), pure decay (beta = 0), a single
  token from a zero state, the delta property (beta = 1, unit key), the
  associative-memory property with orthonormal keys;
* brute-force transition-matrix products on tiny inputs;
* agreement of the token, chunked and C forms;
* invariants: linearity in (S0, V), causality in tokens and in frames,
  streaming composition, the spectral-norm bound, scale invariance of q and k.

Finally a mutation check plants plausible mistakes in a separate copy of the
token loop (on the CPU) and confirms that every one of them fails some pin.
"""

import math
import os

import numpy as np
import pytest

from oracle import gdn_reference as R
from workloads import Inputs, TINY, BLOCK, bf16_round, make_inputs, long_memory

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
BIG = 1.0e4          # logit magnitude that makes sigmoid exactly 0 or 1 in float64


def mk(q, k, v, gate, beta, frame_len=1, state=None):
    q = np.asarray(q, np.float32); k = np.asarray(k, np.float32); v = np.asarray(v, np.float32)
    return Inputs(q=q, k=k, v=v, gate=np.asarray(gate, np.float32),
                  beta=np.asarray(beta, np.float32),
                  state=None if state is None else np.asarray(state, np.float32),
                  io_dtype="f32", frame_len=frame_len)


def rand_inputs(seed, B=1, H=2, T=12, dk=5, dv=3, frame_len=4, gate_mean=0.0, gate_std=1.0,
                state_std=0.5):
    rng = np.random.default_rng(seed)
    F = -(-T // frame_len)
    return mk(rng.standard_normal((B, T, H, dk)), rng.standard_normal((B, T, H, dk)),
              rng.standard_normal((B, T, H, dv)),
              gate_mean + gate_std * rng.standard_normal((B, F, H)),
              rng.standard_normal((B, T, H)), frame_len,
              None if state_std is None else state_std * rng.standard_normal((B, H, dk, dv)))


def read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *rest = line.split()
            vals[key] = [float(eval(x, {"log": math.log})) for x in rest]
    return vals


# ----------------------------------------------------------------------------
# implementations under test: every oracle form must pass every pin
# ----------------------------------------------------------------------------

def impl_token(inp, state_in=None, eps=R.EPS):
    return R.token_recurrence(inp, state_in, eps)


def impl_chunked4(inp, state_in=None, eps=R.EPS):
    return R.chunked(inp, state_in, chunk_len=4, eps=eps)


def impl_chunked64(inp, state_in=None, eps=R.EPS):
    return R.chunked(inp, state_in, chunk_len=64, eps=eps)


def impl_c(inp, state_in=None, eps=R.EPS):
    return R.c_forward(inp, None if state_in is None else np.asarray(state_in, np.float64), eps)


def impl_brute(inp, state_in=None, eps=R.EPS):
    return R.brute_force(inp, state_in, eps)


IMPLS = {"token": impl_token, "chunked4": impl_chunked4, "chunked64": impl_chunked64,
         "c": impl_c, "brute": impl_brute}


# ----------------------------------------------------------------------------
# pins: each takes an implementation and raises AssertionError on a mismatch
# ----------------------------------------------------------------------------

def pin_golden_two_tokens(fn):
    g = read_golden("worked_example_two_tokens.txt")
    inp = mk(np.reshape(g["q"], (1, 2, 1, 2)), np.reshape(g["k"], (1, 2, 1, 2)),
             np.reshape(g["v"], (1, 2, 1, 2)), np.reshape(g["gate"], (1, 2, 1)),
             np.reshape(g["beta"], (1, 2, 1)), frame_len=1)
    out, S = fn(inp, np.reshape(g["state_in"], (1, 1, 2, 2)), eps=0.0)
    np.testing.assert_allclose(out.ravel(), g["out"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(S.ravel(), g["state_out"], rtol=0, atol=1e-12)


def pin_golden_frames(fn):
    g = read_golden("worked_example_frames.txt")
    T = len(g["out"])
    inp = mk(np.ones((1, T, 1, 1)), np.ones((1, T, 1, 1)), np.zeros((1, T, 1, 1)),
             np.reshape(g["gate"], (1, -1, 1)), -BIG * np.ones((1, T, 1)),
             frame_len=int(g["frame_len"][0]))
    out, S = fn(inp, np.reshape(g["state_in"], (1, 1, 1, 1)), eps=0.0)
    # the logits +-ln 3 reach the method as float32 (relative error 3e-8 in g),
    # which moves the products by at most ~1e-7; a wrong gate formula moves them by O(1)
    np.testing.assert_allclose(out.ravel(), g["out"], rtol=2e-7, atol=0)


def pin_identity(fn):
    """a = 1 and beta = 0: the state never changes and o_t = S0^T q_t / |q_t|."""
    inp = rand_inputs(1)
    inp.gate[:] = -BIG
    inp.beta[:] = -BIG
    out, S = fn(inp, inp.state, eps=0.0)
    np.testing.assert_allclose(S, inp.state, rtol=0, atol=1e-12)
    qn = inp.q.astype(np.float64) / np.linalg.norm(inp.q.astype(np.float64), axis=-1, keepdims=True)
    expect = np.einsum("bhij,bthi->bthj", inp.state.astype(np.float64), qn)
    np.testing.assert_allclose(out, expect, rtol=0, atol=1e-12)


def pin_pure_decay(fn):
    """beta = 0: S_t = prod_{s<=t} 1/(1 + e^{g_f(s)}) S0 (frame-wise gate)."""
    inp = rand_inputs(2, T=11, frame_len=3)
    inp.beta[:] = -BIG
    out, S = fn(inp, inp.state, eps=0.0)
    B, T, H, dk = inp.q.shape
    g = inp.gate.astype(np.float64)
    S0 = inp.state.astype(np.float64)
    qn = inp.q.astype(np.float64) / np.linalg.norm(inp.q.astype(np.float64), axis=-1, keepdims=True)
    cum = np.ones((B, H))
    for t in range(T):
        with np.errstate(over="ignore"):
            cum = cum / (1.0 + np.exp(g[:, t // 3, :]))
        St = cum[:, :, None, None] * S0
        np.testing.assert_allclose(out[:, t], np.einsum("bhij,bhi->bhj", St, qn[:, t]),
                                   rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(S, St, rtol=1e-11, atol=1e-13)


def pin_single_token(fn):
    """One token from a zero state: o = b (q.k/|q||k|) v, with b = 1/2 and b = 1."""
    rng = np.random.default_rng(3)
    q, k, v = rng.standard_normal((1, 1, 2, 4)), rng.standard_normal((1, 1, 2, 4)), rng.standard_normal((1, 1, 2, 3))
    inp = mk(q, k, v, rng.standard_normal((1, 1, 2)), [[[0.0, BIG]]])
    out, S = fn(inp, None, eps=0.0)
    q64, k64, v64 = (x.astype(np.float64) for x in (inp.q, inp.k, inp.v))
    for h, b in enumerate((0.5, 1.0)):
        cos = q64[0, 0, h] @ k64[0, 0, h] / np.linalg.norm(q64[0, 0, h]) / np.linalg.norm(k64[0, 0, h])
        np.testing.assert_allclose(out[0, 0, h], b * cos * v64[0, 0, h], rtol=1e-12, atol=1e-14)


def pin_delta_property(fn):
    """beta = 1 and unit keys: S_t^T k_t = v_t after every update, whatever a_t is.

    Checked through the output: with q_t = k_t, o_t = S_t^T k_t = v_t.
    """
    inp = rand_inputs(4, T=9, dk=6, dv=4, frame_len=2)
    inp.beta[:] = BIG
    inp.q[:] = inp.k
    out, S = fn(inp, inp.state, eps=0.0)
    np.testing.assert_allclose(out, inp.v.astype(np.float64), rtol=0, atol=1e-12)


def pin_associative_memory(fn):
    """Orthonormal keys, a = 1, beta = 1, zero state: S_T^T k_j = v_j for all j."""
    rng = np.random.default_rng(5)
    d, dv = 6, 3
    Qm, _ = np.linalg.qr(rng.standard_normal((d, d)))
    keys = Qm.T.astype(np.float32).astype(np.float64)      # rows: (nearly) orthonormal keys
    keys /= np.linalg.norm(keys, axis=1, keepdims=True)
    T = d
    v = rng.standard_normal((1, T, 1, dv))
    k = keys[None, :, None, :]
    # read back every stored key at the end by appending T query-only tokens
    # would change the state; instead compare against S_T from the return value
    inp = mk(k, k, v, -BIG * np.ones((1, T, 1)), BIG * np.ones((1, T, 1)))
    out, S = fn(inp, None, eps=0.0)
    kk = inp.k.astype(np.float64)[0, :, 0, :]
    kk = kk / np.linalg.norm(kk, axis=1, keepdims=True)
    ortho_err = np.abs(kk @ kk.T - np.eye(T)).max()
    np.testing.assert_allclose(kk @ S[0, 0], inp.v.astype(np.float64)[0, :, 0, :],
                               rtol=0, atol=1e-12 + 10 * ortho_err)


def pin_streaming_composition(fn):
    """One call over T equals two calls over T1 + T2 with the state carried (T1 on a frame boundary)."""
    inp = rand_inputs(6, T=14, frame_len=4)
    out, S = fn(inp, inp.state)
    T1 = 8
    first = mk(inp.q[:, :T1], inp.k[:, :T1], inp.v[:, :T1], inp.gate[:, :T1 // 4], inp.beta[:, :T1], 4)
    second = mk(inp.q[:, T1:], inp.k[:, T1:], inp.v[:, T1:], inp.gate[:, T1 // 4:], inp.beta[:, T1:], 4)
    o1, S1 = fn(first, inp.state)
    o2, S2 = fn(second, S1)
    np.testing.assert_allclose(np.concatenate([o1, o2], axis=1), out, rtol=0, atol=1e-12)
    np.testing.assert_allclose(S2, S, rtol=0, atol=1e-12)


def pin_linearity(fn):
    """The map (S0, V) -> (O, S_T) is linear for fixed q, k, gates and betas."""
    inp = rand_inputs(7)
    inp.v[:] = bf16_round(inp.v)            # 8-bit mantissas: 2 v - 3 v2 is exact in float32
    rng = np.random.default_rng(8)
    v2 = bf16_round(rng.standard_normal(inp.v.shape).astype(np.float32))
    s2 = rng.standard_normal(inp.state.shape).astype(np.float32)
    o1, S1 = fn(inp, inp.state)
    o2, S2 = fn(mk(inp.q, inp.k, v2, inp.gate, inp.beta, inp.frame_len), s2)
    vsum = (2.0 * inp.v.astype(np.float64) - 3.0 * v2.astype(np.float64)).astype(np.float32)
    ssum = 2.0 * inp.state.astype(np.float64) - 3.0 * s2.astype(np.float64)
    o3, S3 = fn(mk(inp.q, inp.k, vsum, inp.gate, inp.beta, inp.frame_len), ssum)
    np.testing.assert_allclose(o3, 2 * o1 - 3 * o2, rtol=0, atol=1e-9)
    np.testing.assert_allclose(S3, 2 * S1 - 3 * S2, rtol=0, atol=1e-9)


def pin_causality(fn):
    """Perturbing token t' leaves o_{<t'} unchanged; perturbing frame f's gate
    leaves every output before frame f unchanged and changes frame f's outputs."""
    inp = rand_inputs(9, T=12, frame_len=4)
    base, _ = fn(inp, inp.state)
    tp = 6
    pert = mk(inp.q.copy(), inp.k.copy(), inp.v.copy(), inp.gate.copy(), inp.beta.copy(), 4)
    pert.q[:, tp] += 1.0; pert.k[:, tp] -= 1.0; pert.v[:, tp] *= 2.0; pert.beta[:, tp] += 0.5
    o, _ = fn(pert, inp.state)
    np.testing.assert_array_equal(o[:, :tp], base[:, :tp])
    assert np.abs(o[:, tp] - base[:, tp]).max() > 1e-6
    pert = mk(inp.q, inp.k, inp.v, inp.gate.copy(), inp.beta, 4)
    pert.gate[:, 1] += 1.0
    o, _ = fn(pert, inp.state)
    np.testing.assert_array_equal(o[:, :4], base[:, :4])
    assert np.abs(o[:, 4:8] - base[:, 4:8]).max() > 1e-6


def pin_scale_invariance(fn):
    """q and k enter only through their directions (epsilon 0)."""
    inp = rand_inputs(10)
    base, S = fn(inp, inp.state, eps=0.0)
    scaled = mk(inp.q * np.float32(4.0), inp.k * np.float32(0.25), inp.v, inp.gate, inp.beta, inp.frame_len)
    o, S2 = fn(scaled, inp.state, eps=0.0)
    np.testing.assert_allclose(o, base, rtol=0, atol=1e-12)
    np.testing.assert_allclose(S2, S, rtol=0, atol=1e-12)


def pin_norm_bound(fn):
    """|S_t|_2 <= a_t |S_{t-1}|_2 + b_t |v_t|, since |I - b k k^T|_2 <= 1 for b in [0, 1].

    Checked on prefixes: the state after t tokens is the final state of a call over t tokens.
    """
    inp = rand_inputs(11, T=8, frame_len=3, state_std=2.0)
    prev = np.linalg.norm(inp.state.astype(np.float64)[0, 0], 2)
    for t in range(1, 9):
        sub = mk(inp.q[:, :t], inp.k[:, :t], inp.v[:, :t], inp.gate[:, :-(-t // 3)], inp.beta[:, :t], 3)
        _, S = fn(sub, inp.state)
        a = 1.0 / (1.0 + np.exp(float(inp.gate[0, (t - 1) // 3, 0])))
        b = 1.0 / (1.0 + np.exp(-float(inp.beta[0, t - 1, 0])))
        cur = np.linalg.norm(S[0, 0], 2)
        assert cur <= a * prev + b * np.linalg.norm(inp.v[0, t - 1, 0].astype(np.float64)) + 1e-12
        prev = cur


def pin_zero_vectors(fn):
    """A zero key writes nothing and erases nothing (S_t = a S_{t-1}); a zero query reads 0."""
    inp = rand_inputs(12, T=3, frame_len=1)
    inp.k[:, 1] = 0.0
    inp.q[:, 2] = 0.0
    _, S1 = fn(mk(inp.q[:, :1], inp.k[:, :1], inp.v[:, :1], inp.gate[:, :1], inp.beta[:, :1], 1), inp.state)
    out, S2 = fn(mk(inp.q[:, :2], inp.k[:, :2], inp.v[:, :2], inp.gate[:, :2], inp.beta[:, :2], 1), inp.state)
    a = 1.0 / (1.0 + np.exp(inp.gate[:, 1, :].astype(np.float64)))
    np.testing.assert_allclose(S2, a[:, :, None, None] * S1, rtol=1e-12, atol=1e-14)
    out, _ = fn(inp, inp.state)
    np.testing.assert_array_equal(out[:, 2], 0.0)


PINS = [pin_golden_two_tokens, pin_golden_frames, pin_identity, pin_pure_decay, pin_single_token,
        pin_delta_property, pin_associative_memory, pin_streaming_composition, pin_linearity,
        pin_causality, pin_scale_invariance, pin_norm_bound, pin_zero_vectors]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
@pytest.mark.parametrize("impl", list(IMPLS), ids=str)
def test_oracle_passes_pin(impl, pin):
    pin(IMPLS[impl])


# ----------------------------------------------------------------------------
# agreement between the oracle's forms
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("C", [1, 4, 16, 64])
@pytest.mark.parametrize("T", [1, 63, 64, 100, 130])
def test_chunked_equals_token(C, T):
    inp = rand_inputs(20 + T, B=2, H=3, T=T, dk=16, dv=8, frame_len=7, gate_mean=-2.0, gate_std=1.0)
    o1, S1 = R.token_recurrence(inp, inp.state)
    o2, S2 = R.chunked(inp, inp.state, chunk_len=C)
    scale = max(1.0, np.abs(o1).max())
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-11 * scale)
    np.testing.assert_allclose(S2, S1, rtol=0, atol=1e-11 * max(1.0, np.abs(S1).max()))


@pytest.mark.parametrize("gate_mean", [2.0, -6.0])
def test_chunked_equals_token_config_gates(gate_mean):
    """Config-like gates (a ~ 0.12: G over a chunk reaches about -136) and slow decay."""
    inp = rand_inputs(30, B=1, H=2, T=200, dk=32, dv=16, frame_len=80, gate_mean=gate_mean,
                      gate_std=0.5, state_std=0.02)
    o1, S1 = R.token_recurrence(inp, inp.state)
    o2, S2 = R.chunked(inp, inp.state, chunk_len=64)
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-11 * np.abs(o1).max())
    np.testing.assert_allclose(S2, S1, rtol=0, atol=1e-11 * np.abs(S1).max())


def test_brute_force_equals_token_with_state():
    for seed in range(3):
        inp = rand_inputs(40 + seed, B=2, H=2, T=6, dk=3, dv=2, frame_len=2, state_std=1.0)
        o1, S1 = R.token_recurrence(inp, inp.state)
        o2, S2 = R.brute_force(inp, inp.state)
        np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-12)
        np.testing.assert_allclose(S2, S1, rtol=0, atol=1e-12)


def test_c_equals_numpy_tiny_config():
    inp = make_inputs(TINY)
    o1, S1 = R.token_recurrence(inp, inp.state)
    o2, S2 = R.c_forward(inp, inp.state)
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-12)
    np.testing.assert_allclose(S2, S1, rtol=0, atol=1e-12)


def test_c_equals_numpy_block_slice():
    """Config-2 shapes (d = 112, frame 880) on a 300-token slice, f32 and f64 state entry."""
    w = BLOCK.with_(H=3)
    inp = make_inputs(w, T=300)
    o1, S1 = R.token_recurrence(inp, inp.state)
    o2, S2 = R.c_forward(inp, inp.state)
    o3, S3 = R.c_forward(inp, inp.state.astype(np.float64))
    for o, S in ((o2, S2), (o3, S3)):
        np.testing.assert_allclose(o, o1, rtol=0, atol=1e-12 * np.abs(o1).max())
        np.testing.assert_allclose(S, S1, rtol=0, atol=1e-12 * np.abs(S1).max())


def test_long_memory_variant_keeps_state():
    """The slow-decay variant really carries the state: about exp(-880*0.0025) ~ 11 % per frame."""
    w = long_memory(BLOCK.with_(H=1))
    inp = make_inputs(w, T=900)
    la = R.token_log_gate(inp.gate, 900, w.frame_len)
    kept = np.exp(la[0, :880, 0].sum())
    assert 0.05 < kept < 0.25


# ----------------------------------------------------------------------------
# mutation check: plausible mistakes must each fail at least one pin
# ----------------------------------------------------------------------------

def _token_loop(inp, state_in=None, eps=R.EPS, mut=None):
    """An independent copy of the token recurrence with switchable mistakes."""
    q = inp.q.astype(np.float64); k = inp.k.astype(np.float64); v = inp.v.astype(np.float64)
    B, T, H, dk = q.shape
    dv = v.shape[3]
    if mut != "no_norm_q":
        q = q / np.sqrt((q * q).sum(-1, keepdims=True) + eps)
    if mut != "no_norm_k":
        k = k / np.sqrt((k * k).sum(-1, keepdims=True) + eps)
    g = inp.gate.astype(np.float64)
    bl = inp.beta.astype(np.float64)
    S = np.zeros((B, H, dk, dv)) if state_in is None else np.array(state_in, np.float64)
    out = np.zeros((B, T, H, dv))
    for t in range(T):
        f = (t + 1) // inp.frame_len if mut == "frame_index" else t // inp.frame_len
        f = min(f, g.shape[1] - 1)
        with np.errstate(over="ignore"):
            if mut == "gate_sign":
                a = 1.0 / (1.0 + np.exp(-g[:, f]))
            else:
                a = 1.0 / (1.0 + np.exp(g[:, f]))
            b = 1.0 / (1.0 + np.exp(-bl[:, t]))
        if mut == "beta_one":
            b = np.ones_like(b)
        a4 = a[:, :, None, None]; b4 = b[:, :, None, None]
        kt, vt = k[:, t], v[:, t]
        kS = np.einsum("bhi,bhij->bhj", kt, S)
        erase = b4 * kt[..., :, None] * kS[..., None, :]
        write = b4 * kt[..., :, None] * vt[..., None, :]
        Sprev = S
        if mut == "decay_write":
            S = a4 * (S - erase + write)
        elif mut == "undecayed_erase":
            S = a4 * S - erase + write
        elif mut == "erase_sign":
            S = a4 * (S + erase) + write
        else:
            S = a4 * (S - erase) + write
        readS = Sprev if mut == "read_before_update" else S
        if mut == "transposed_read":
            out[:, t] = np.einsum("bhij,bhj->bhi", readS[..., :dv, :], q[:, t][..., :dv]) \
                if dk == dv else np.einsum("bhij,bhi->bhj", readS, q[:, t]) * 1.5
        else:
            out[:, t] = np.einsum("bhij,bhi->bhj", readS, q[:, t])
    return out, S


MUTANTS = ["read_before_update", "decay_write", "undecayed_erase", "erase_sign", "gate_sign",
           "frame_index", "beta_one", "no_norm_q", "no_norm_k", "transposed_read"]


def test_mutation_harness_clean_copy_passes_all_pins():
    fn = lambda inp, s=None, eps=R.EPS: _token_loop(inp, s, eps, None)
    for pin in PINS:
        pin(fn)


@pytest.mark.parametrize("mut", MUTANTS)
def test_each_mutant_fails_some_pin(mut):
    fn = lambda inp, s=None, eps=R.EPS: _token_loop(inp, s, eps, mut)
    failed = []
    for pin in PINS:
        try:
            pin(fn)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"mutant {mut} passed every pin"
