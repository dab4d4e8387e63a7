"""GPU parity of the fp8 (e4m3) input variant, gdn_forward_fp8, against the float64
oracle run on the widened values (q = e4m3(q8), k = e4m3(k8), v = v_scale *
e4m3(v8)).  Widening e4m3 to bf16 is exact, so the bars are the bf16 ones:
max-abs <= 2e-2 and relative L2 <= 5e-3 on out and on the final state.

Cases: ragged and single-token sequences, several head sizes, a scale that is
not a power of two (small sizes, float64 numpy oracle), the SANA-WM block,
clip241 and minute-scale layers, long-memory gates, a streaming step with the
state in place, T = 0 (the state passes through), and the argument checks.
Outputs are NaN-filled with guard bands.
"""

import numpy as np
import pytest

from oracle import gdn_reference as R
from workloads import BLOCK, CLIP241, MINUTE, draw, long_memory, make_fp8_inputs, to_fp8

from gpu_util import assert_bf16_parity, f32_device, host

pytestmark = pytest.mark.gpu


def upload8(x8, device):
    import torch
    u8 = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
    return u8(x8.q8), u8(x8.k8), u8(x8.v8), f32_device(x8.gate, device), f32_device(x8.beta, device)


def run_fp8(x8, device, state_in=None, want_state=True):
    import torch
    import hybrid_linear_attention_frame_b200 as G
    q8, k8, v8, g, b = upload8(x8, device)
    Bn, T, H, dk = x8.q8.shape
    dv = x8.v8.shape[3]
    guard = 64
    out_buf = torch.full((Bn * T * H * dv + 2 * guard,), float("nan"), dtype=torch.bfloat16, device=device)
    out_buf[:guard] = 7.0
    out_buf[-guard:] = 7.0
    out = out_buf[guard:-guard]
    st = torch.full((Bn, H, dk, dv), float("nan"), dtype=torch.float32, device=device) if want_state else None
    s_in = None if state_in is None else f32_device(state_in, device)
    G.gdn_forward_fp8(q8, k8, v8, x8.v_scale, g, b, s_in, st, out, Bn, H, T, dk, dv, x8.frame_len, 64)
    torch.cuda.synchronize()
    assert G.gdn_get_last_device_status() == G.GDN_OK
    assert bool((out_buf[:guard] == 7.0).all()) and bool((out_buf[-guard:] == 7.0).all()), "write outside out"
    o = host(out).reshape(Bn, T, H, dv)
    assert not np.isnan(o).any()
    return o, (None if st is None else host(st))


def oracle(x8, state_in):
    w = R.widen_fp8(x8)
    Bn, T, H, _ = x8.q8.shape
    if Bn * T * H <= 20000 or not float(np.log2(x8.v_scale)).is_integer():
        return R.token_recurrence(w, state_in)
    return R.c_forward(w, state_in)          # power-of-two scale: the float32 inputs are exact


def check(x8, device, what, with_state=True):
    s_in = x8.state if with_state else None
    o, s = run_fp8(x8, device, s_in)
    ro, rs = oracle(x8, s_in)
    assert_bf16_parity(o, ro, what + " out")
    assert_bf16_parity(s, rs, what + " state")


def small_cases():
    rng = np.random.Generator(np.random.PCG64(91))
    mk = lambda B, H, T, dk, dv, fl, gm, gs, st: to_fp8(draw(rng, B, H, T, dk, dv, fl, "f32", gm, gs, state_std=st))
    return {
        "T1 d16": mk(1, 1, 1, 16, 16, 1, 0.0, 1.0, 0.3),
        "T65 d112": mk(1, 2, 65, 112, 112, 880, 0.0, 1.0, 0.3),
        "T63 d64 B2H3": mk(2, 3, 63, 64, 64, 10, 0.0, 1.0, None),
        "T700 d112 B2H20": mk(2, 20, 700, 112, 112, 100, 0.0, 1.5, 0.3),
        "T300 d48x80": mk(1, 3, 300, 48, 80, 7, 0.0, 1.0, 0.3),
    }


@pytest.mark.parametrize("name", sorted(small_cases()))
def test_fp8_parity_small(cuda, name):
    x8 = small_cases()[name]
    check(x8, cuda, name, with_state=x8.state is not None)


def test_fp8_scale_not_a_power_of_two(cuda):
    rng = np.random.Generator(np.random.PCG64(92))
    x8 = to_fp8(draw(rng, 1, 4, 200, 112, 112, 40, "f32", 0.0, 1.0, state_std=0.3), v_scale=0.0123)
    check(x8, cuda, "scale 0.0123")


@pytest.mark.parametrize("w", [BLOCK, CLIP241, long_memory(CLIP241)], ids=["block", "clip241", "clip241_longmem"])
def test_fp8_parity_configs(cuda, w):
    x8 = make_fp8_inputs(w)
    check(x8, cuda, w.name, with_state=x8.state is not None)


@pytest.mark.slow
def test_fp8_parity_minute_layer(cuda):
    x8 = make_fp8_inputs(MINUTE)
    check(x8, cuda, "minute", with_state=False)


def test_fp8_streaming_step_in_place(cuda):
    """Three blocks with the state carried in place (state_in == state_out)."""
    import torch
    import hybrid_linear_attention_frame_b200 as G
    rng = np.random.Generator(np.random.PCG64(93))
    Bn, H, T, d = 2, 20, 2640, 112
    s0 = (0.02 * rng.standard_normal((Bn, H, d, d))).astype(np.float32)
    st = f32_device(s0, cuda).contiguous()
    ref = s0.astype(np.float64)
    for n in range(3):
        x8 = to_fp8(draw(rng, Bn, H, T, d, d, 880, "f32", 2.0, 0.5))
        q8, k8, v8, g, b = upload8(x8, cuda)
        out = torch.empty((Bn, T, H, d), dtype=torch.bfloat16, device=cuda)
        G.gdn_forward_fp8(q8, k8, v8, x8.v_scale, g, b, st, st, out, Bn, H, T, d, d, 880, 64)
        torch.cuda.synchronize()
        assert G.gdn_get_last_device_status() == G.GDN_OK
        ro, ref = R.c_forward(R.widen_fp8(x8), ref)
        assert_bf16_parity(host(out), ro, f"block {n} out")
    assert_bf16_parity(host(st), ref, "final state")


def test_fp8_zero_tokens_passes_the_state(cuda):
    import torch
    import hybrid_linear_attention_frame_b200 as G
    rng = np.random.Generator(np.random.PCG64(94))
    x8 = to_fp8(draw(rng, 1, 2, 1, 112, 112, 880, "f32", 2.0, 0.5, state_std=0.3))
    q8, k8, v8, g, b = upload8(x8, cuda)
    s_in = f32_device(x8.state, cuda)
    s_out = torch.full_like(s_in, float("nan"))
    out = torch.full((16,), 3.0, dtype=torch.bfloat16, device=cuda)
    assert G.gdn_forward_fp8(q8, k8, v8, 1.0, g, b, s_in, s_out, out, 1, 2, 0, 112, 112, 880, 64) == G.GDN_OK
    torch.cuda.synchronize()
    assert torch.equal(s_out, s_in)
    assert bool((out == 3.0).all())


def test_fp8_argument_checks(cuda):
    import torch
    import hybrid_linear_attention_frame_b200 as G
    rng = np.random.Generator(np.random.PCG64(95))
    x8 = to_fp8(draw(rng, 1, 2, 64, 128, 128, 64, "f32", 2.0, 0.5))
    q8, k8, v8, g, b = upload8(x8, cuda)
    out = torch.empty((1, 64, 2, 128), dtype=torch.bfloat16, device=cuda)
    args = (g, b, None, None, out, 1, 2, 64)
    # d 128: not taken by the e4m3 kernel
    assert G.gdn_forward_fp8(q8, k8, v8, 1.0, *args, 128, 128, 64, 64, check=False) == G.GDN_ERR_UNSUPPORTED
    # d 112 buffers carved from the same tensors
    q, k, v = q8.view(-1)[:64 * 2 * 112], k8.view(-1)[:64 * 2 * 112], v8.view(-1)[:64 * 2 * 112]
    o = out.view(-1)[:64 * 2 * 112]
    a = (g, b, None, None, o, 1, 2, 64, 112, 112, 64)
    assert G.gdn_forward_fp8(q, k, v, 1.0, *a, 32, check=False) == G.GDN_ERR_UNSUPPORTED       # chunk 32
    assert G.gdn_forward_fp8(q, k, v, -1.0, *a, 64, check=False) == G.GDN_ERR_INVALID_ARG      # negative scale
    assert G.gdn_forward_fp8(q, k, v, float("nan"), *a, 64, check=False) == G.GDN_ERR_INVALID_ARG
    assert G.gdn_forward_fp8(q8.view(-1)[1:], k, v, 1.0, *a, 64, check=False) == G.GDN_ERR_INVALID_ARG  # misaligned
    # out overlapping v (out is bf16: twice the bytes of v)
    vo = torch.empty(64 * 2 * 112 * 3, dtype=torch.uint8, device=cuda)
    n = 64 * 2 * 112
    assert G.gdn_forward_fp8(q, k, vo[:n], 1.0, g, b, None, None, vo[n - 16:], 1, 2, 64, 112, 112, 64, 64,
                             check=False) == G.GDN_ERR_INVALID_ARG
    torch.cuda.synchronize()
