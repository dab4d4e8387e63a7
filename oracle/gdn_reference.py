"""Float64 CPU oracle for the frame-wise Gated DeltaNet forward pass.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg may import this module or load the C
library it wraps.  Nothing here is shared with the CUDA library.

The method (fixed in writing, since the SANA-WM pages name "frame-wise Gated
DeltaNet" in the sglang cookbook's architecture table but print no formula):
per batch entry and head,

    S_t = a_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T,   o_t = S_t^T q_t,

q and k L2-normalised per token (x / sqrt(sum x^2 + eps), eps = 1e-6),
beta_t = sigmoid(beta logit of token t), and a = exp(-softplus(gate logit of
frame f)) shared by all tokens of latent frame f = t // frame_len.  The other
reading of "frame-wise" (inputs with gate_mode 1) applies a_f once, at the first
token of frame f, and a_t = 1 at the frame's other tokens.

Three independent float64 forms live here:

* ``token_recurrence`` -- the recurrence above, one token at a time (numpy,
  vectorised over batch and heads only).
* ``chunked`` -- the chunk-parallel (WY / UT) form of the same recurrence,
  derived from it: within a chunk with cumulative log-gates G_i,
      (I + L) E = diag(beta) (V - diag(e^G) K S_0),  L strictly lower,
      L_ij = beta_i (k_i . k_j) e^(G_i - G_j),
      O   = diag(e^G) Q S_0 + (Q K^T o e^(G_i - G_j) [j <= i]) E,
      S_C = e^(G_C) S_0 + (diag(e^(G_C - G)) K)^T E.
  This is the chunking of the (gated) delta rule published by Yang et al.
  ("Parallelizing Linear Transformers with the Delta Rule over Sequence
  Length", 2024; "Gated Delta Networks", 2024), re-derived from the
  recurrence; it is used only to check the algebra a chunked kernel relies on.
* ``brute_force`` -- explicit products of the per-token transition matrices
  M_t = a_t (I - beta_t k_t k_t^T), for tiny sizes.

and a ctypes wrapper, ``c_forward``, for the C token recurrence in
``gdn_oracle.c`` (OpenMP over chains), used at full sizes.

The dense checkpoint's bidirectional GDN (sglang cookbook SANA-WM page,
dense-bidirectional section) is not defined on the pages; it is fixed here as
the sum of the forward scan and the same rule run from the last token to the
first, both from a zero state, every token keeping its own q, k, v, beta and the
gate of its own frame (at every token):

    R_t = a_t (I - beta_t k_t k_t^T) R_{t+1} + beta_t k_t v_t^T,  R_T = 0,
    o_t = S_t^T q_t + R_t^T q_t.

``token_recurrence_backward`` is that backward loop, ``bidirectional`` the sum,
``c_bidirectional`` the C form of the sum.

The fp8 input variant (the FlashDreams SANA-WM streaming runner page ships fp8
precision modes without a scheme) is read as: q, k, v given as OCP e4m3 bytes,
v with one float scale, v = v_scale * e4m3(v8); the layer is the recurrence
above on those values.  ``decode_e4m3`` writes out the e4m3 format and
``widen_fp8`` turns such inputs into the float64 values every form here takes.
"""

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

EPS = 1e-6
_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libgdn_oracle.so")
_SRC_PATH = os.path.join(_HERE, "gdn_oracle.c")


# ----------------------------------------------------------------------------
# elementwise definitions
# ----------------------------------------------------------------------------


def decode_e4m3(codes):
    """OCP e4m3 bytes -> float64: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa
    bits; exponent field 0 holds the subnormals m/8 * 2^-6, field 1..15 the normals
    (1 + m/8) * 2^(e-7); the one code with all of exponent and mantissa set
    (0x7F, 0xFF) is NaN and there are no infinities, so the largest value is 448."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c >> 7, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    mag = np.where((e == 0xF) & (m == 7), np.nan, mag)
    return sign * mag


class Widened:
    """fp8 inputs as the float64 values of the layer (the fields the forms here read)."""

    def __init__(self, x8):
        self.q = decode_e4m3(x8.q8)
        self.k = decode_e4m3(x8.k8)
        self.v = float(x8.v_scale) * decode_e4m3(x8.v8)
        self.gate = x8.gate
        self.beta = x8.beta
        self.state = x8.state
        self.frame_len = x8.frame_len
        self.gate_mode = getattr(x8, "gate_mode", GATE_EVERY_TOKEN)
        self.io_dtype = "f32"


def widen_fp8(x8):
    """q = e4m3(q8), k = e4m3(k8), v = v_scale * e4m3(v8), the rest unchanged."""
    return Widened(x8)

def softplus(x):
    """log(1 + e^x), computed without overflow."""
    x = np.asarray(x, dtype=np.float64)
    return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))


def sigmoid(x):
    x = np.asarray(x, dtype=np.float64)
    with np.errstate(over="ignore"):          # exp(-x) -> inf gives exactly 0
        return 1.0 / (1.0 + np.exp(-x))


def l2_normalise(x, eps=EPS):
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)


GATE_EVERY_TOKEN = 0     # a_f at every token of frame f
GATE_FRAME_START = 1     # a_f once, at the first token of frame f (a_t = 1 elsewhere)


def token_log_gate(gate, T, frame_len, gate_mode=GATE_EVERY_TOKEN):
    """Per-token log-gate log a_t, f(t) = t // frame_len.

    gate_mode 0: log a_t = -softplus(gate[f(t)]) at every token ("frame-wise" read
    as one gate shared by the frame's tokens).  gate_mode 1: the same value at the
    first token of each frame (t % frame_len == 0) and 0 at the others ("frame-wise"
    read as one decay per frame step).
    gate: [B, F, H]  ->  [B, T, H] float64.
    """
    t = np.arange(T)
    la = -softplus(np.asarray(gate, dtype=np.float64)[:, t // frame_len, :])
    if gate_mode == GATE_FRAME_START:
        la[:, t % frame_len != 0, :] = 0.0
    elif gate_mode != GATE_EVERY_TOKEN:
        raise ValueError(f"unknown gate_mode {gate_mode}")
    return la


def _prep(inp, eps):
    B, T, H, dk = inp.q.shape
    qn = l2_normalise(inp.q, eps)
    kn = l2_normalise(inp.k, eps)
    v = np.asarray(inp.v, dtype=np.float64)
    la = token_log_gate(inp.gate, T, inp.frame_len, getattr(inp, "gate_mode", GATE_EVERY_TOKEN))
    bt = sigmoid(inp.beta)
    return qn, kn, v, la, bt


def _init_state(inp, state_in):
    B, T, H, dk = inp.q.shape
    dv = inp.v.shape[3]
    if state_in is None:
        return np.zeros((B, H, dk, dv))
    return np.array(state_in, dtype=np.float64, copy=True)


# ----------------------------------------------------------------------------
# token recurrence
# ----------------------------------------------------------------------------

def token_recurrence(inp, state_in=None, eps=EPS, return_states=False):
    """The recurrence one token at a time.  Returns (out [B,T,H,d_v], S_T [B,H,d_k,d_v]).

    With ``return_states`` also returns every S_t as [T, B, H, d_k, d_v].
    """
    qn, kn, v, la, bt = _prep(inp, eps)
    S = _init_state(inp, state_in)
    B, T, H, _ = qn.shape
    out = np.zeros(v.shape)
    states = [] if return_states else None
    for t in range(T):
        a = np.exp(la[:, t, :])[:, :, None, None]            # [B,H,1,1]
        b = bt[:, t, :][:, :, None, None]
        k_t = kn[:, t, :, :]                                 # [B,H,dk]
        v_t = v[:, t, :, :]                                  # [B,H,dv]
        kS = np.einsum("bhi,bhij->bhj", k_t, S)              # k^T S_{t-1}
        S = a * (S - b * k_t[..., :, None] * kS[..., None, :]) \
            + b * k_t[..., :, None] * v_t[..., None, :]
        out[:, t] = np.einsum("bhij,bhi->bhj", S, qn[:, t])  # S_t^T q
        if return_states:
            states.append(S.copy())
    if return_states:
        return out, S, np.stack(states) if states else np.zeros((0,) + S.shape)
    return out, S


def token_recurrence_backward(inp, eps=EPS):
    """The same rule run from the last token to the first, from a zero state:
    R_t = a_t (I - beta_t k_t k_t^T) R_{t+1} + beta_t k_t v_t^T, output R_t^T q_t.
    Token t keeps its own frame's gate.  Returns out [B,T,H,d_v]."""
    if getattr(inp, "gate_mode", GATE_EVERY_TOKEN) != GATE_EVERY_TOKEN:
        raise ValueError("the backward scan takes the gate at every token only")
    qn, kn, v, la, bt = _prep(inp, eps)
    B, T, H, dk = qn.shape
    R = np.zeros((B, H, dk, v.shape[3]))
    out = np.zeros(v.shape)
    for t in range(T - 1, -1, -1):
        a = np.exp(la[:, t, :])[:, :, None, None]
        b = bt[:, t, :][:, :, None, None]
        k_t = kn[:, t, :, :]
        kR = np.einsum("bhi,bhij->bhj", k_t, R)              # k^T R_{t+1}
        R = a * (R - b * k_t[..., :, None] * kR[..., None, :]) \
            + b * k_t[..., :, None] * v[:, t, :, :][..., None, :]
        out[:, t] = np.einsum("bhij,bhi->bhj", R, qn[:, t])
    return out


def bidirectional(inp, eps=EPS):
    """Forward scan plus backward scan, both from a zero state.  Returns out [B,T,H,d_v]."""
    fwd, _ = token_recurrence(inp, None, eps)
    return fwd + token_recurrence_backward(inp, eps)


# ----------------------------------------------------------------------------
# chunked (WY / UT) form
# ----------------------------------------------------------------------------

def chunked(inp, state_in=None, chunk_len=64, eps=EPS):
    """Chunk-parallel form of the same recurrence (float64, for checking the algebra)."""
    qn, kn, v, la, bt = _prep(inp, eps)
    S = _init_state(inp, state_in)
    B, T, H, dk = qn.shape
    out = np.zeros(v.shape)
    for c0 in range(0, T, chunk_len):
        c1 = min(c0 + chunk_len, T)
        L = c1 - c0
        Q = qn[:, c0:c1].transpose(0, 2, 1, 3)              # [B,H,L,dk]
        K = kn[:, c0:c1].transpose(0, 2, 1, 3)
        V = v[:, c0:c1].transpose(0, 2, 1, 3)               # [B,H,L,dv]
        beta = bt[:, c0:c1].transpose(0, 2, 1)              # [B,H,L]
        G = np.cumsum(la[:, c0:c1].transpose(0, 2, 1), axis=-1)   # G_i = sum_{s<=i} log a_s
        diff = G[..., :, None] - G[..., None, :]            # G_i - G_j
        incl = np.tril(np.ones((L, L), dtype=bool))
        strict = np.tril(np.ones((L, L), dtype=bool), -1)
        # decay ratios only where i >= j (never exp of a positive difference)
        Gam = np.where(incl, np.exp(np.where(incl, diff, 0.0)), 0.0)
        KK = K @ np.swapaxes(K, -1, -2)
        A = np.where(strict, beta[..., :, None] * KK * Gam, 0.0)
        eye = np.eye(L)
        Tm = np.linalg.solve(eye + A, np.broadcast_to(eye, A.shape) * beta[..., None, :])
        gam = np.exp(G)[..., None]                          # e^{G_i}
        W = Tm @ (gam * K)
        U = Tm @ V
        E = U - W @ S
        P = (Q @ np.swapaxes(K, -1, -2)) * Gam
        O = gam * (Q @ S) + P @ E
        out[:, c0:c1] = O.transpose(0, 2, 1, 3)
        gC = G[..., -1:]                                     # G at the chunk's last token
        Kd = np.exp(gC - G)[..., None] * K
        S = np.exp(gC)[..., None] * S + np.swapaxes(Kd, -1, -2) @ E
    return out, S


# ----------------------------------------------------------------------------
# brute force
# ----------------------------------------------------------------------------

def brute_force(inp, state_in=None, eps=EPS):
    """Explicit transition products, for tiny T and d only.

    S_t = (M_t ... M_1) S_0 + sum_j (M_t ... M_{j+1}) beta_j k_j v_j^T,
    M_t = a_t (I - beta_t k_t k_t^T), o_t = S_t^T q_t.
    """
    qn, kn, v, la, bt = _prep(inp, eps)
    S0 = _init_state(inp, state_in)
    B, T, H, dk = qn.shape
    dv = v.shape[3]
    out = np.zeros(v.shape)
    ST = np.zeros_like(S0)
    for b in range(B):
        for h in range(H):
            M = [np.exp(la[b, t, h]) * (np.eye(dk) - bt[b, t, h] * np.outer(kn[b, t, h], kn[b, t, h]))
                 for t in range(T)]
            for t in range(T):
                prod = np.eye(dk)
                for s in range(t, -1, -1):
                    prod = prod @ M[s]                       # M_t ... M_s
                St = prod @ S0[b, h]
                for j in range(t + 1):
                    Pj = np.eye(dk)
                    for s in range(t, j, -1):
                        Pj = Pj @ M[s]                       # M_t ... M_{j+1}
                    St = St + bt[b, j, h] * Pj @ np.outer(kn[b, j, h], v[b, j, h])
                out[b, t, h] = St.T @ qn[b, t, h]
                if t == T - 1:
                    ST[b, h] = St
            if T == 0:
                ST[b, h] = S0[b, h]
    return out, ST


# ----------------------------------------------------------------------------
# C token recurrence (OpenMP over chains)
# ----------------------------------------------------------------------------

_lib = None


def build(force: bool = False) -> str:
    """Compile ``gdn_oracle.c`` into ``libgdn_oracle.so`` beside it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or \
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC_PATH):
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", _LIB_PATH, _SRC_PATH, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        fp = ctypes.POINTER(ctypes.c_float)
        dp = ctypes.POINTER(ctypes.c_double)
        args = [fp, fp, fp, fp, fp, None, dp, dp] + [ctypes.c_int] * 6 + [ctypes.c_double, ctypes.c_int,
                                                                          ctypes.c_int]
        f = lib.gdn_oracle_forward
        f.argtypes = args[:5] + [fp] + args[6:]
        f.restype = ctypes.c_int
        g = lib.gdn_oracle_forward_f64state
        g.argtypes = args[:5] + [dp] + args[6:]
        g.restype = ctypes.c_int
        h = lib.gdn_oracle_bidirectional
        h.argtypes = [fp] * 5 + [dp] + [ctypes.c_int] * 6 + [ctypes.c_double, ctypes.c_int]
        h.restype = ctypes.c_int
        lib.gdn_oracle_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def max_threads() -> int:
    return int(_load().gdn_oracle_max_threads())


def c_forward(inp, state_in=None, eps=EPS, n_threads=0, want_state=True):
    """C token recurrence.  state_in may be float32 or float64 (kept in float64)."""
    lib = _load()
    B, T, H, dk = inp.q.shape
    dv = inp.v.shape[3]
    fp = ctypes.POINTER(ctypes.c_float)
    dp = ctypes.POINTER(ctypes.c_double)

    def f32(a):
        return np.ascontiguousarray(a, dtype=np.float32)

    q, k, v, g, b = f32(inp.q), f32(inp.k), f32(inp.v), f32(inp.gate), f32(inp.beta)
    out = np.empty((B, T, H, dv), dtype=np.float64)
    st_out = np.empty((B, H, dk, dv), dtype=np.float64) if want_state else None
    st_out_p = st_out.ctypes.data_as(dp) if want_state else ctypes.cast(None, dp)
    common = (q.ctypes.data_as(fp), k.ctypes.data_as(fp), v.ctypes.data_as(fp),
              g.ctypes.data_as(fp), b.ctypes.data_as(fp))
    dims = (B, H, T, dk, dv, inp.frame_len, float(eps), int(n_threads),
            int(getattr(inp, "gate_mode", GATE_EVERY_TOKEN)))
    if state_in is not None and np.asarray(state_in).dtype == np.float64:
        s = np.ascontiguousarray(state_in, dtype=np.float64)
        rc = lib.gdn_oracle_forward_f64state(*common, s.ctypes.data_as(dp), st_out_p,
                                             out.ctypes.data_as(dp), *dims)
    else:
        s = None if state_in is None else f32(state_in)
        sp = ctypes.cast(None, fp) if s is None else s.ctypes.data_as(fp)
        rc = lib.gdn_oracle_forward(*common, sp, st_out_p, out.ctypes.data_as(dp), *dims)
    if rc != 0:
        raise RuntimeError("gdn_oracle_forward failed")
    return out, st_out


def c_bidirectional(inp, eps=EPS, n_threads=0):
    """C form of ``bidirectional`` (forward plus backward scan from zero states)."""
    if getattr(inp, "gate_mode", GATE_EVERY_TOKEN) != GATE_EVERY_TOKEN:
        raise ValueError("the bidirectional form takes the gate at every token only")
    lib = _load()
    B, T, H, dk = inp.q.shape
    dv = inp.v.shape[3]
    fp = ctypes.POINTER(ctypes.c_float)
    dp = ctypes.POINTER(ctypes.c_double)

    def f32(a):
        return np.ascontiguousarray(a, dtype=np.float32)

    q, k, v, g, b = f32(inp.q), f32(inp.k), f32(inp.v), f32(inp.gate), f32(inp.beta)
    out = np.empty((B, T, H, dv), dtype=np.float64)
    rc = lib.gdn_oracle_bidirectional(q.ctypes.data_as(fp), k.ctypes.data_as(fp), v.ctypes.data_as(fp),
                                      g.ctypes.data_as(fp), b.ctypes.data_as(fp), out.ctypes.data_as(dp),
                                      B, H, T, dk, dv, inp.frame_len, float(eps), int(n_threads))
    if rc != 0:
        raise RuntimeError("gdn_oracle_bidirectional failed")
    return out
