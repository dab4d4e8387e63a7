"""Failure detection on the device without a fault: every wait in the kernels is
bounded, and a wait that runs out makes the kernel stop, record GDN_ERR_TIMEOUT and
return, leaving the context usable.

The test shortens the bound to 1 ns through gdn_set_wait_limit_ns, so that the
first wait that does not succeed at once gives up (nothing is broken: the
producer is simply slower than the bound).  Under a bound below 1 ms the mbarrier
waits poll without a suspend hint and read the clock on every poll, and the ring
kernel's counter waits read it every ~1 us, so every kernel reports the timeout:
the ring kernel (gdn_forward_ws), the sequence-parallel kernel (gdn_forward at
d 112, and its e4m3-input instance through gdn_forward_fp8), the fused chunk
kernel (gdn_forward at d 128) and the softmax-attention kernel
(gdn_softmax_attention).  Each kernel then
drains the copies and MMAs it has in flight and returns.  After each such call
the default bound is restored and a normal call must match the untouched
reference outputs bit for bit.
"""

import numpy as np
import pytest

from workloads import draw, to_fp8

from gpu_util import f32_device, upload

pytestmark = pytest.mark.gpu


def _inputs(d, fp8=False):
    rng = np.random.Generator(np.random.PCG64(77))
    # 2 x 20 chains of 700 tokens (at d 112 a ring of 7 x 20 CTAs)
    inp = draw(rng, 2, 20, 700, d, d, 100, "f32" if fp8 else "bf16", gate_mean=0.0, gate_std=1.5, state_std=0.3)
    return to_fp8(inp) if fp8 else inp


def _upload_fp8(x8, device):
    import torch
    u8 = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
    return u8(x8.q8), u8(x8.k8), u8(x8.v8), f32_device(x8.gate, device), f32_device(x8.beta, device)


def _run(G, entry, tensors, inp, ws):
    import torch
    q, k, v, g, b, s_in = tensors
    Bn, T, H, dk = q.shape
    dv = v.shape[3]
    o = torch.full(tuple(v.shape), float("nan"), dtype=torch.bfloat16, device=v.device)
    s = torch.full((Bn, H, dk, dv), float("nan"), dtype=torch.float32, device=v.device)
    if entry == "ws":
        G.gdn_forward_ws(q, k, v, g, b, s_in, s, o, Bn, H, T, dk, dv, inp.frame_len, 64, ws)
    elif entry == "fp8":
        G.gdn_forward_fp8(q, k, v, inp.v_scale, g, b, s_in, s, o, Bn, H, T, dk, dv, inp.frame_len, 64)
    elif entry == "attn":
        # the softmax-attention kernel (no state: s stays as filled)
        s.zero_()
        G.gdn_softmax_attention(q, k, v, o, Bn, H, T, dk, dv, inp.frame_len, 3, 2, 1)
    else:
        G.gdn_forward(q, k, v, g, b, s_in, s, o, Bn, H, T, dk, dv, inp.frame_len, 64)
    return o, s, G.gdn_get_last_device_status()


@pytest.mark.parametrize("entry,d,path", [("ws", 112, None), ("plain", 112, 2), ("plain", 128, 1), ("fp8", 112, 2),
                                          ("attn", 112, None)],
                         ids=["ring", "sequence_parallel", "fused_d128", "sequence_parallel_e4m3", "softmax_attention"])
def test_wait_timeout_is_reported_and_context_recovers(cuda, entry, d, path):
    import torch
    import hybrid_linear_attention_frame_b200 as G
    if path is not None:
        assert G.gdn_bf16_path(d, d, 64) == path
    inp = _inputs(d, fp8=entry == "fp8")
    q, k, v, g, b = _upload_fp8(inp, cuda) if entry == "fp8" else upload(inp, cuda)
    s_in = f32_device(inp.state, cuda)
    Bn, T, H, dk = q.shape
    dv = v.shape[3]
    ws = G.workspace(Bn, H, T, dk, dv, 64, cuda)
    tensors = (q, k, v, g, b, s_in)

    ref_o, ref_s, st = _run(G, entry, tensors, inp, ws)
    assert st == G.GDN_OK

    try:
        assert G.gdn_set_wait_limit_ns(1) == G.GDN_OK
        for _ in range(3):
            _, _, st = _run(G, entry, tensors, inp, ws)
            assert st == G.GDN_ERR_TIMEOUT, G.status_string(st)
            print(f"{entry}: status under a 1 ns bound: {G.status_string(st)}")
    finally:
        G.gdn_set_wait_limit_ns(0)

    # the status word was cleared by the read; the next calls run normally
    for _ in range(2):
        o, s, st = _run(G, entry, tensors, inp, ws)
        assert st == G.GDN_OK
        assert torch.equal(o, ref_o)
        assert torch.equal(s, ref_s)
    torch.cuda.synchronize()
