"""GPU parity of gdn_softmax_attention (chunk-causal softmax attention with the rolling
KV cache of SANA-WM's softmax layers) against the float64 oracle.  Bars as for the
bf16 GDN path: max-abs <= 2e-2 and relative L2 <= 5e-3 on the output.

Cases: blocks shorter than a 128-query tile (every tile spans several blocks, each
row with its own key set), blocks longer than a tile, no sink, no cache, two sink
frames, d_k != d_v, a single token, a sub-tile sequence, several batch entries and
heads; at the clip241 and minute-scale shapes, sampled queries (block starts and
ends, the partial last block) computed one by one.  Outputs are NaN-filled with
guard bands first.
"""

import numpy as np
import pytest

from oracle import attention_reference as A
from workloads import CLIP241, MINUTE, draw, make_inputs

from gpu_util import assert_bf16_parity, host, upload

pytestmark = pytest.mark.gpu


def run_attn(inp, device, fl, fpb=3, nc=2, sk=1):
    import torch
    import hybrid_linear_attention_frame_b200 as G
    q, k, v, _, _ = upload(inp, device)
    Bn, T, H, dk = inp.q.shape
    dv = inp.v.shape[3]
    guard = 64
    n_out = Bn * T * H * dv
    buf = torch.full((n_out + 2 * guard,), float("nan"), dtype=torch.bfloat16, device=device)
    buf[:guard] = 7.0
    buf[-guard:] = 7.0
    out = buf[guard:guard + n_out]
    G.gdn_softmax_attention(q, k, v, out, Bn, H, T, dk, dv, fl, fpb, nc, sk)
    torch.cuda.synchronize()
    assert G.gdn_get_last_device_status() == G.GDN_OK
    assert torch.all(buf[:guard] == 7.0) and torch.all(buf[-guard:] == 7.0), "guard band overwritten"
    o = host(out).reshape(Bn, T, H, dv)
    assert not np.isnan(o).any(), "output not fully written"
    return o


SEED = 41

# (B, H, T, d_k, d_v, frame_len, frames_per_block, cached, sink_frames)
CASES = {
    "blocks shorter than a tile": (1, 2, 700, 112, 112, 40, 1, 2, 1),
    "blocks of 300, two batch entries": (2, 3, 1000, 112, 112, 100, 3, 2, 1),
    "no sink": (1, 2, 900, 112, 112, 50, 3, 2, 0),
    "no cache": (1, 2, 800, 112, 112, 60, 2, 0, 1),
    "two sink frames, one cached block": (1, 2, 1100, 112, 112, 70, 2, 1, 2),
    "d_k 96, d_v 128": (1, 2, 600, 96, 128, 50, 3, 2, 1),
    "d 80 and 128, ragged tile": (1, 1, 333, 128, 80, 30, 3, 2, 1),
    "single token": (1, 4, 1, 112, 112, 880, 3, 2, 1),
    "sub-tile sequence": (2, 2, 57, 112, 112, 10, 3, 2, 1),
    "sink inside the window, long blocks": (1, 2, 1300, 112, 112, 200, 3, 2, 1),
    "two whole query tiles": (1, 2, 256, 112, 112, 40, 2, 1, 1),
    "one row in the second query tile": (1, 2, 129, 112, 112, 20, 3, 2, 1),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_attention_parity(cuda, name):
    Bn, H, T, dk, dv, fl, fpb, nc, sk = CASES[name]
    rng = np.random.Generator(np.random.PCG64(SEED + T))
    inp = draw(rng, Bn, H, T, dk, dv, fl, "bf16", 0.0, 1.0)
    o = run_attn(inp, cuda, fl, fpb, nc, sk)
    ref = A.chunk_causal_attention(inp.q, inp.k, inp.v, fl, fpb, nc, sk)
    assert_bf16_parity(o, ref, f"attention {name}")


def test_attention_large_scores(cuda):
    """Scores far from zero (q scaled up): the reference maximum must move and the
    accumulator be rescaled, without overflow."""
    rng = np.random.Generator(np.random.PCG64(SEED + 1))
    inp = draw(rng, 1, 2, 900, 112, 112, 50, "bf16", 0.0, 1.0)
    from workloads import bf16_round
    inp.q[:] = bf16_round(inp.q * 6.0)
    o = run_attn(inp, cuda, 50, 3, 2, 1)
    ref = A.chunk_causal_attention(inp.q, inp.k, inp.v, 50, 3, 2, 1)
    assert_bf16_parity(o, ref, "attention large scores")


def sampled_check(inp, device, what, n_samples=160):
    fl = inp.frame_len
    o = run_attn(inp, device, fl, 3, 2, 1)
    Bn, T, H, _ = inp.q.shape
    bl = 3 * fl
    rng = np.random.default_rng(SEED + 2)
    picks = set()
    for b0 in range(0, T, bl):                      # every block's first and last query
        picks.add((0, b0, int(rng.integers(H))))
        picks.add((0, min(T, b0 + bl) - 1, int(rng.integers(H))))
    picks.update((0, T - 1, h) for h in range(H))
    while len(picks) < n_samples + 2 * (-(-T // bl)):
        picks.add((0, int(rng.integers(T)), int(rng.integers(H))))
    picks = sorted(picks)
    got = np.stack([o[b, t, h] for (b, t, h) in picks])
    ref = np.stack([A.attention_one_query(inp.q, inp.k, inp.v, b, t, h, fl, 3, 2, 1) for (b, t, h) in picks])
    assert_bf16_parity(got, ref, f"{what} ({len(picks)} sampled queries)")


def test_attention_clip241_sampled(cuda):
    sampled_check(make_inputs(CLIP241), cuda, "attention clip241")


def test_attention_minute_sampled(cuda):
    sampled_check(make_inputs(MINUTE), cuda, "attention minute")


def test_attention_argument_checks(cuda):
    import torch
    import hybrid_linear_attention_frame_b200 as G
    x = torch.zeros((1, 64, 2, 112), dtype=torch.bfloat16, device=cuda)
    out = torch.empty_like(x)
    assert G.gdn_softmax_attention(x, x, x, out, 1, 2, 64, 112, 112, 16, check=False) == G.GDN_OK
    assert G.gdn_softmax_attention(x, x, x, x, 1, 2, 64, 112, 112, 16, check=False) == G.GDN_ERR_INVALID_ARG
    assert G.gdn_softmax_attention(x, x, x, out, 1, 2, 64, 64, 64, 16, check=False) == G.GDN_ERR_UNSUPPORTED
    assert G.gdn_softmax_attention(x, x, x, out, 1, 2, 64, 112, 112, 0, check=False) == G.GDN_ERR_INVALID_ARG
    assert G.gdn_softmax_attention(x, x, x, out, 1, 2, 0, 112, 112, 16, check=False) == G.GDN_OK
    torch.cuda.synchronize()
    assert G.gdn_get_last_device_status() == G.GDN_OK
