"""Float64 CPU oracle for SANA-WM's chunk-causal softmax attention layer.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg may import this module.  Nothing here is
shared with the CUDA library.

What it computes.  SANA-WM's DiT interleaves the frame-wise GDN layers with a
softmax-attention block every 4 blocks (sglang cookbook SANA-WM page, section 1
architecture table).  In streaming generation the video is produced in blocks of
``num_frame_per_block`` = 3 latent frames; the softmax layers keep a rolling KV
cache of the last ``num_cached_blocks`` = 2 blocks plus ``sink_size`` = 1 sink
frame (same page, pipeline-configuration table).  Over a whole sequence of T tokens
(frame_len tokens per latent frame, block_len = frames_per_block * frame_len) this
is, per batch entry and head,

    o_t = sum_{s in K(t)} softmax_s(q_t . k_s / sqrt(d_k)) v_s,

    K(t) = [0, sink_len)  union  [max(0, b - cached) * block_len, min(T, (b + 1) * block_len)),

with b = t // block_len and sink_len = sink_frames * frame_len: the sink frames,
the cached blocks and the whole current block (keys after t inside the current
block included: "chunk-causal" is causal across blocks, full within one).  The
scale 1/sqrt(d_k) is the usual one; the pages print none.

``chunk_causal_attention`` evaluates this block by block (``attention_block``: all
queries of a block share K); ``attention_one_query`` evaluates one query, for
sampled checks of full-size outputs.
"""

import math

import numpy as np


def block_keys(b, T, frame_len, frames_per_block=3, cached_blocks=2, sink_frames=1):
    """Sorted key token indices of query block b."""
    bl = frames_per_block * frame_len
    lo = max(0, b - cached_blocks) * bl
    hi = min(T, (b + 1) * bl)
    sink = min(T, sink_frames * frame_len)
    if lo <= sink:
        return np.arange(0, hi)
    return np.concatenate([np.arange(0, sink), np.arange(lo, hi)])


def _softmax_rows(scores):
    m = np.max(scores, axis=-1, keepdims=True)
    e = np.exp(scores - m)
    return e / np.sum(e, axis=-1, keepdims=True)


def attention_block(q, k, v, b, frame_len, frames_per_block=3, cached_blocks=2, sink_frames=1, scale=None):
    """Outputs of query block b alone: [B, len(block), H, d_v] (float64)."""
    B, T, H, dk = q.shape
    sc = 1.0 / math.sqrt(dk) if scale is None else scale
    bl = frames_per_block * frame_len
    t0, t1 = b * bl, min(T, (b + 1) * bl)
    keys = block_keys(b, T, frame_len, frames_per_block, cached_blocks, sink_frames)
    qb = np.asarray(q[:, t0:t1], np.float64).transpose(0, 2, 1, 3)          # [B, H, t, d_k]
    kb = np.asarray(k[:, keys], np.float64).transpose(0, 2, 3, 1)           # [B, H, d_k, s]
    vb = np.asarray(v[:, keys], np.float64).transpose(0, 2, 1, 3)           # [B, H, s, d_v]
    p = _softmax_rows((qb @ kb) * sc)                                       # [B, H, t, s]
    return (p @ vb).transpose(0, 2, 1, 3)


def chunk_causal_attention(q, k, v, frame_len, frames_per_block=3, cached_blocks=2, sink_frames=1,
                           scale=None):
    """q, k [B, T, H, d_k], v [B, T, H, d_v] -> out [B, T, H, d_v] (float64)."""
    B, T, H, dk = np.shape(q)
    bl = frames_per_block * frame_len
    out = np.zeros(np.shape(v)[:3] + (np.shape(v)[3],))
    for b in range(-(-T // bl)):
        out[:, b * bl:min(T, (b + 1) * bl)] = attention_block(q, k, v, b, frame_len, frames_per_block,
                                                              cached_blocks, sink_frames, scale)
    return out


def attention_one_query(q, k, v, bi, t, h, frame_len, frames_per_block=3, cached_blocks=2, sink_frames=1,
                        scale=None):
    """o_t of batch entry bi and head h alone (float64 vector of d_v)."""
    T, dk = q.shape[1], q.shape[3]
    sc = 1.0 / math.sqrt(dk) if scale is None else scale
    keys = block_keys(t // (frames_per_block * frame_len), T, frame_len, frames_per_block, cached_blocks,
                      sink_frames)
    qt = np.asarray(q[bi, t, h], np.float64)
    s = (np.asarray(k[bi, keys, h], np.float64) @ qt) * sc
    p = _softmax_rows(s[None, :])[0]
    return p @ np.asarray(v[bi, keys, h], np.float64)
