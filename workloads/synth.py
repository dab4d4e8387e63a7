"""Seeded synthetic inputs shared by the oracle tests, the GPU tests and the bench.

This module holds no arithmetic of the method. It draws standard normals from
numpy's ``Generator(PCG64(seed))`` in float32, in the fixed order
q, k, v, gate logits, beta logits, initial state, scales and shifts them to the
workload's distributions, and rounds the bf16 tensors to bf16 with
round-to-nearest-even.  Both sides of a parity test receive exactly the same
values: the GPU side the bf16 bit patterns, the oracle the same values widened
to float32 (exact).

Layouts (row-major, contiguous):
  q, k      [B, T, H, d_k]
  v         [B, T, H, d_v]
  gate      [B, ceil(T / frame_len), H]   one logit per latent frame and head
  beta      [B, T, H]                     one logit per token and head
  state     [B, H, d_k, d_v]              float32
"""

from dataclasses import dataclass
from typing import Optional

import numpy as np

from .configs import Workload


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    r = (u >> np.uint32(16)) & np.uint32(1)
    u = u + np.uint32(0x7FFF) + r
    u &= np.uint32(0xFFFF0000)
    return u.view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Upper 16 bits of float32 values that are already bf16-representable."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return (x.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


@dataclass
class Inputs:
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    gate: np.ndarray
    beta: np.ndarray
    state: Optional[np.ndarray]
    io_dtype: str
    frame_len: int
    # where the frame's gate applies: 0 = at every token of the frame, 1 = once, at
    # the frame's first token (the two readings of "frame-wise"; see the oracle)
    gate_mode: int = 0

    @property
    def shape(self):
        B, T, H, dk = self.q.shape
        return B, H, T, dk, self.v.shape[3]


def _normal(rng, shape, mean=0.0, std=1.0):
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    if mean != 0.0:
        x += np.float32(mean)
    return x


def draw(rng: np.random.Generator, B: int, H: int, T: int, d_k: int, d_v: int,
         frame_len: int, io_dtype: str, gate_mean: float, gate_std: float,
         beta_mean: float = 0.0, beta_std: float = 1.0,
         state_std: Optional[float] = None) -> Inputs:
    """Draw one set of inputs from ``rng`` in the fixed order q, k, v, gate, beta, state."""
    F = -(-T // frame_len)
    q = _normal(rng, (B, T, H, d_k))
    k = _normal(rng, (B, T, H, d_k))
    v = _normal(rng, (B, T, H, d_v))
    gate = _normal(rng, (B, F, H), gate_mean, gate_std)
    beta = _normal(rng, (B, T, H), beta_mean, beta_std)
    state = None
    if state_std is not None:
        state = _normal(rng, (B, H, d_k, d_v), 0.0, state_std)
    if io_dtype == "bf16":
        q, k, v = bf16_round(q), bf16_round(k), bf16_round(v)
    elif io_dtype != "f32":
        raise ValueError(io_dtype)
    return Inputs(q, k, v, gate, beta, state, io_dtype, frame_len)


def make_inputs(w: Workload, T: Optional[int] = None, seed: Optional[int] = None) -> Inputs:
    """Inputs of one call of workload ``w`` (optionally with another T or seed)."""
    rng = np.random.Generator(np.random.PCG64(w.seed if seed is None else seed))
    return draw(rng, w.B, w.H, w.T if T is None else T, w.d_k, w.d_v, w.frame_len,
                w.io_dtype, w.gate_mean, w.gate_std, w.beta_mean, w.beta_std, w.state_std)


def make_session_blocks(w: Workload, n_blocks: Optional[int] = None):
    """Batched streaming: session s draws from seed ``session_seed_base + s``.

    Per session the generator first draws the initial state [H, d_k, d_v]
    (N(0, state_std)), then each block's q, k, v, gate, beta in turn.  The
    sessions are stacked along B.  Returns (initial_state, [Inputs per block]);
    the per-block Inputs carry ``state=None``.
    """
    n_blocks = w.blocks if n_blocks is None else n_blocks
    base = w.session_seed_base if w.session_seed_base is not None else 1000
    rngs = [np.random.Generator(np.random.PCG64(base + s)) for s in range(w.B)]
    std = w.state_std if w.state_std is not None else 0.0
    state0 = np.stack([_normal(r, (w.H, w.d_k, w.d_v), 0.0, std) for r in rngs])
    blocks = []
    for _ in range(n_blocks):
        parts = [draw(r, 1, w.H, w.T, w.d_k, w.d_v, w.frame_len, w.io_dtype,
                      w.gate_mean, w.gate_std, w.beta_mean, w.beta_std, None) for r in rngs]
        blocks.append(Inputs(
            q=np.concatenate([p.q for p in parts]), k=np.concatenate([p.k for p in parts]),
            v=np.concatenate([p.v for p in parts]), gate=np.concatenate([p.gate for p in parts]),
            beta=np.concatenate([p.beta for p in parts]), state=None,
            io_dtype=w.io_dtype, frame_len=w.frame_len))
    return state0, blocks


# ---------------------------------------------------------------- e4m3 inputs
#
# The fp8 input variant takes q, k and v as OCP e4m3 bytes.  Producing those bytes
# is the caller's quantisation, not part of the layer, so it lives here with the
# other input generation: round-to-nearest-even from the float32 draws, saturating
# at +-448 (the largest finite e4m3 value).  q and k are encoded as drawn; v is
# divided by one power-of-two scale first, so that max |v| / scale <= 448 and the
# scaled values stay exactly representable in float32.


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """float32 -> e4m3 codes (uint8): nearest value, ties to even, saturating."""
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    neg = np.signbit(x)
    m = np.minimum(np.abs(x), 448.0)
    # exponent of the binade (subnormals share the quantum of the lowest binade)
    e = np.clip(np.floor(np.log2(np.maximum(m, 2.0 ** -10))), -6, 8)
    quantum = np.exp2(e - 3)
    qv = np.minimum(np.round(m / quantum) * quantum, 448.0)     # np.round: ties to even
    sub = qv < 2.0 ** -6
    e2 = np.floor(np.log2(np.where(sub, 1.0, qv)))
    mant = np.where(sub, qv * 512.0, (qv / np.exp2(e2) - 1.0) * 8.0)
    expo = np.where(sub, 0.0, e2 + 7.0)
    code = (expo.astype(np.int64) << 3) | mant.astype(np.int64)
    return (code | (neg.astype(np.int64) << 7)).astype(np.uint8)


def v_scale_for(v: np.ndarray) -> float:
    """The power-of-two scale that maps max |v| into the e4m3 range."""
    amax = float(np.max(np.abs(v))) if v.size else 0.0
    if amax == 0.0:
        return 1.0
    return float(2.0 ** np.ceil(np.log2(amax / 448.0)))


@dataclass
class Fp8Inputs:
    q8: np.ndarray          # uint8 e4m3 codes [B, T, H, d_k]
    k8: np.ndarray          # uint8 e4m3 codes [B, T, H, d_k]
    v8: np.ndarray          # uint8 e4m3 codes [B, T, H, d_v]
    v_scale: float          # v = v_scale * e4m3(v8)
    gate: np.ndarray
    beta: np.ndarray
    state: Optional[np.ndarray]
    frame_len: int
    gate_mode: int = 0


def to_fp8(inp: Inputs, v_scale: Optional[float] = None) -> Fp8Inputs:
    """Encode float32 draws (io_dtype 'f32') as e4m3 inputs."""
    if inp.io_dtype != "f32":
        raise ValueError("encode the float32 draws, not rounded copies")
    s = v_scale_for(inp.v) if v_scale is None else float(v_scale)
    v = (inp.v.astype(np.float64) / s).astype(np.float32)
    return Fp8Inputs(e4m3_encode(inp.q), e4m3_encode(inp.k), e4m3_encode(v), s,
                     inp.gate, inp.beta, inp.state, inp.frame_len, inp.gate_mode)


def make_fp8_inputs(w: Workload, T: Optional[int] = None, seed: Optional[int] = None) -> Fp8Inputs:
    """e4m3 inputs of one call of workload ``w``: the same draws as ``make_inputs``
    (before bf16 rounding), encoded."""
    rng = np.random.Generator(np.random.PCG64(w.seed if seed is None else seed))
    inp = draw(rng, w.B, w.H, w.T if T is None else T, w.d_k, w.d_v, w.frame_len,
               "f32", w.gate_mean, w.gate_std, w.beta_mean, w.beta_std, w.state_std)
    return to_fp8(inp)
