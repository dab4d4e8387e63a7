"""Pins of the chunk-causal softmax attention oracle (the softmax layers of SANA-WM's
hybrid stack with their rolling KV cache: sglang cookbook SANA-WM page, section 1
architecture table and pipeline-configuration table).  The key sets are checked
against a simulation of the streaming cache written independently of the oracle's
range arithmetic; the arithmetic against a hand-derived example, PyTorch's
scaled_dot_product_attention, closed forms and invariants.  Mistakes planted in a
copy of the oracle must fail a pin.  CPU only.
"""

import math

import numpy as np
import pytest

from oracle import attention_reference as A

from test_oracle_pins import read_golden


def cache_simulation_mask(T, frame_len, frames_per_block, cached, sink_frames):
    """Stream the sequence block by block through a rolling KV cache: the sink holds
    the first sink_frames frames ever seen, the cache the last `cached` blocks; a
    block's queries see the sink, the cache and the block itself.  Returns [T, T]."""
    bl = frames_per_block * frame_len
    sink_len = sink_frames * frame_len
    mask = np.zeros((T, T), dtype=bool)
    sink, cache = [], []
    for b0 in range(0, T, bl):
        block = list(range(b0, min(T, b0 + bl)))
        visible = set(sink) | set(block)
        for old in cache:
            visible |= set(old)
        for t in block:
            mask[t, sorted(visible)] = True
        for t in block:
            if len(sink) < sink_len:
                sink.append(t)
        cache.append(block)
        if len(cache) > cached:
            cache.pop(0)
    return mask


def rand_qkv(seed, B=2, T=23, H=2, dk=5, dv=3):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((B, T, H, dk)), rng.standard_normal((B, T, H, dk)),
            rng.standard_normal((B, T, H, dv)))


GEOMS = [(1, 2, 1, 1), (2, 3, 2, 1), (3, 1, 2, 2), (2, 2, 0, 1), (1, 3, 2, 0), (4, 3, 2, 1)]


def impl_oracle(q, k, v, fl, fpb, nc, sk, scale=None):
    return A.chunk_causal_attention(q, k, v, fl, fpb, nc, sk, scale)


# ----------------------------------------------------------------------------
# pins: each takes an implementation with the oracle's signature
# ----------------------------------------------------------------------------

def pin_golden(fn):
    g = read_golden("worked_example_attention.txt")
    T = len(g["out"])
    q = np.ones((1, T, 1, 1))
    k = np.reshape(np.asarray(g["k"], np.float32), (1, T, 1, 1))      # ln 3 reaches the method as float32
    v = np.reshape(g["v"], (1, T, 1, 1))
    out = fn(q, k, v, int(g["frame_len"][0]), int(g["frames_per_block"][0]), int(g["cached"][0]),
             int(g["sink"][0]))
    np.testing.assert_allclose(out.ravel(), g["out"], rtol=1e-7, atol=0)


def pin_uniform_scores_average_the_cache(fn):
    """q = 0: every visible key has the same weight, so o_t is the mean of v over the
    keys the streaming cache shows to t."""
    for (fl, fpb, nc, sk) in GEOMS:
        T = 23
        q, k, v = rand_qkv(1, T=T)
        q[:] = 0.0
        out = fn(q, k, v, fl, fpb, nc, sk)
        mask = cache_simulation_mask(T, fl, fpb, nc, sk)
        expect = np.einsum("ts,bshd->bthd", mask / mask.sum(axis=1, keepdims=True), v)
        np.testing.assert_allclose(out, expect, rtol=0, atol=1e-12)


def pin_library_sdpa(fn):
    """Against torch's scaled_dot_product_attention (float64, CPU) given the cache
    simulation's mask."""
    import torch
    import torch.nn.functional as F
    for (fl, fpb, nc, sk) in GEOMS:
        T = 23
        q, k, v = rand_qkv(2, T=T, dk=6, dv=4)
        out = fn(q, k, v, fl, fpb, nc, sk)
        mask = torch.from_numpy(cache_simulation_mask(T, fl, fpb, nc, sk))
        tq, tk, tv = (torch.from_numpy(x).permute(0, 2, 1, 3) for x in (q, k, v))   # [B, H, T, d]
        ref = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask).permute(0, 2, 1, 3).numpy()
        np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def pin_single_token(fn):
    q, k, v = rand_qkv(3, T=1)
    np.testing.assert_allclose(fn(q, k, v, 4, 3, 2, 1), v, rtol=0, atol=1e-15)


def pin_key_shift_invariance(fn):
    """Adding one vector c to every key adds q_t . c to every score of query t."""
    q, k, v = rand_qkv(4, T=19)
    c = np.random.default_rng(5).standard_normal(k.shape[-1])
    np.testing.assert_allclose(fn(q, k + c, v, 2, 2, 1, 1), fn(q, k, v, 2, 2, 1, 1), rtol=0, atol=1e-12)


def pin_value_affine(fn):
    """The weights sum to one: v -> a v + c gives o -> a o + c."""
    q, k, v = rand_qkv(6, T=17)
    np.testing.assert_allclose(fn(q, k, 2.5 * v - 0.75, 3, 2, 2, 1), 2.5 * fn(q, k, v, 3, 2, 2, 1) - 0.75,
                               rtol=0, atol=1e-12)


def pin_scale(fn):
    """The scores are q . k / sqrt(d_k): dividing q by sqrt(d_k) and passing scale 1 agrees."""
    q, k, v = rand_qkv(7, T=15, dk=9)
    np.testing.assert_allclose(fn(q / 3.0, k, v, 2, 2, 1, 1, scale=1.0), fn(q, k, v, 2, 2, 1, 1), rtol=0,
                               atol=1e-12)


def pin_locality(fn):
    """Keys and values outside K(t) do not reach o_t; inside they do."""
    T, fl, fpb, nc, sk = 30, 2, 2, 1, 1         # blocks of 4 tokens; sink = tokens 0, 1
    q, k, v = rand_qkv(8, T=T)
    base = fn(q, k, v, fl, fpb, nc, sk)
    k2, v2 = k.copy(), v.copy()
    k2[:, 9] += 1.0                               # block 2
    v2[:, 9] -= 2.0
    out = fn(q, k2, v2, fl, fpb, nc, sk)
    changed = np.any(np.abs(out - base) > 1e-12, axis=(0, 2, 3))
    expect = np.zeros(T, dtype=bool)
    expect[8:16] = True                           # blocks 2 (own) and 3 (caches block 2)
    np.testing.assert_array_equal(changed, expect)


PINS = [pin_golden, pin_uniform_scores_average_the_cache, pin_library_sdpa, pin_single_token,
        pin_key_shift_invariance, pin_value_affine, pin_scale, pin_locality]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_attention_pin(pin):
    pin(impl_oracle)


def test_one_query_matches_block_form():
    q, k, v = rand_qkv(9, B=2, T=41, H=3, dk=7, dv=5)
    out = A.chunk_causal_attention(q, k, v, 3, 3, 2, 1)
    for (bi, t, h) in [(0, 0, 0), (1, 8, 2), (0, 9, 1), (1, 26, 0), (0, 40, 2)]:
        np.testing.assert_allclose(A.attention_one_query(q, k, v, bi, t, h, 3, 3, 2, 1), out[bi, t, h],
                                   rtol=0, atol=1e-13)


def test_key_sets_match_cache_simulation():
    for (fl, fpb, nc, sk) in GEOMS + [(880, 3, 2, 1)]:
        T = 23 if fl < 100 else 880 * 10 + 17
        bl = fl * fpb
        mask = cache_simulation_mask(T, fl, fpb, nc, sk) if T < 2000 else None
        for b in range(-(-T // bl)):
            keys = A.block_keys(b, T, fl, fpb, nc, sk)
            assert np.all(np.diff(keys) > 0)
            if mask is not None:
                for t in range(b * bl, min(T, (b + 1) * bl)):
                    np.testing.assert_array_equal(np.flatnonzero(mask[t]), keys)
            else:
                lo = max(0, b - nc) * bl
                assert len(keys) == min(T, (b + 1) * bl) - lo + (fl * sk if lo > fl * sk else lo)


# ----------------------------------------------------------------------------
# planted mistakes
# ----------------------------------------------------------------------------

def _mutant(kind):
    def fn(q, k, v, fl, fpb, nc, sk, scale=None):
        q = np.asarray(q, np.float64); k = np.asarray(k, np.float64); v = np.asarray(v, np.float64)
        B, T, H, dk = q.shape
        sc = (1.0 / math.sqrt(dk) if scale is None else scale) if kind != "no_scale" else 1.0
        bl = fpb * fl
        out = np.zeros(v.shape)
        for b in range(-(-T // bl)):
            t0, t1 = b * bl, min(T, (b + 1) * bl)
            nc_eff = nc + 1 if kind == "window_one_block_long" else nc
            sk_eff = 0 if kind == "no_sink" else sk
            keys = A.block_keys(b, T, fl, fpb, nc_eff, sk_eff)
            s = np.einsum("bthd,bshd->bhts", q[:, t0:t1], k[:, keys]) * sc
            if kind == "causal_within_block":
                tq = np.arange(t0, t1)[:, None]
                s = np.where(keys[None, :] <= tq, s, -np.inf)
            m = np.max(s, axis=-1, keepdims=True)
            e = np.exp(s - m)
            p = e / (np.sum(e, axis=-1, keepdims=True) if kind != "no_normalise" else 1.0)
            out[:, t0:t1] = np.einsum("bhts,bshd->bthd", p, v[:, keys])
        return out
    return fn


@pytest.mark.parametrize("kind", ["no_scale", "window_one_block_long", "no_sink", "causal_within_block",
                                  "no_normalise"])
def test_planted_mistake_fails_a_pin(kind):
    fn = _mutant(kind)
    failed = []
    for pin in PINS:
        try:
            pin(fn)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"mistake {kind} passes every pin"
