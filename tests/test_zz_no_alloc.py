"""The allocation-free entry point gdn_forward_static_ws (the ring kept in a static
device array inside the library) against gdn_forward_ws with a caller workspace.
Both run the same kernel on the same inputs, so results must be identical, and stay
so on a second call in a row (the static array keeps the previous call's contents,
which must not matter).  It also checks what the entry point is for: after a first
call has set it up on the device, further calls allocate no device memory, neither
through the CUDA driver (free bytes on the device) nor through PyTorch's allocator.
Collected last on purpose: it must pass alone and after every other test of the
session.
"""

import numpy as np
import pytest

from workloads import BLOCK, draw, long_memory, make_inputs

from gpu_util import f32_device, upload

pytestmark = pytest.mark.gpu


def _cases():
    rng = np.random.Generator(np.random.PCG64(2024))
    return [
        ("block, state in and out", make_inputs(BLOCK), True),
        ("block long-memory, zero state", make_inputs(long_memory(BLOCK)), False),
        ("40 chains, several per group of CTAs",
         draw(rng, 2, 20, 700, 112, 112, 100, "bf16", gate_mean=0.0, gate_std=1.5, state_std=0.3), True),
        ("d 64: a size served without a ring", draw(rng, 1, 3, 200, 64, 64, 50, "bf16", 0.0, 1.0, state_std=0.3), True),
    ]


@pytest.mark.parametrize("case", range(4))
def test_static_scratch_matches_workspace_entry_two_calls(cuda, case):
    import torch
    import hybrid_linear_attention_frame_b200 as G
    what, inp, with_state = _cases()[case]
    q, k, v, g, b = upload(inp, cuda)
    Bn, T, H, dk = inp.q.shape
    dv = inp.v.shape[3]
    s_in = f32_device(inp.state, cuda) if with_state else None
    ws = G.workspace(Bn, H, T, dk, dv, 64, cuda)
    ref_o = torch.empty_like(v)
    ref_s = torch.empty((Bn, H, dk, dv), dtype=torch.float32, device=cuda)
    G.gdn_forward_ws(q, k, v, g, b, s_in, ref_s, ref_o, Bn, H, T, dk, dv, inp.frame_len, 64, ws)
    def call_and_compare(call):
        o = torch.full_like(v, float("nan"))
        s = torch.full_like(ref_s, float("nan"))
        G.gdn_forward_static_ws(q, k, v, g, b, s_in, s, o, Bn, H, T, dk, dv, inp.frame_len, 64)
        torch.cuda.synchronize()
        assert G.gdn_get_last_device_status() == G.GDN_OK
        assert torch.equal(o, ref_o), f"{what}: out differs on call {call}"
        assert torch.equal(s, ref_s), f"{what}: state differs on call {call}"
        return o, s

    keep = call_and_compare(0)          # first call on the device: sets up the scratch address
    del keep
    torch.cuda.synchronize()
    free0, alloc0 = torch.cuda.mem_get_info(cuda)[0], torch.cuda.memory_allocated(cuda)
    o = torch.empty_like(v)
    s = torch.empty_like(ref_s)
    free1, alloc1 = torch.cuda.mem_get_info(cuda)[0], torch.cuda.memory_allocated(cuda)
    for call in (1, 2):
        o.fill_(float("nan"))
        s.fill_(float("nan"))
        G.gdn_forward_static_ws(q, k, v, g, b, s_in, s, o, Bn, H, T, dk, dv, inp.frame_len, 64)
        torch.cuda.synchronize()
        assert G.gdn_get_last_device_status() == G.GDN_OK
        assert torch.equal(o, ref_o), f"{what}: out differs on call {call}"
        assert torch.equal(s, ref_s), f"{what}: state differs on call {call}"
        assert torch.cuda.memory_allocated(cuda) == alloc1, f"{what}: PyTorch allocation on call {call}"
        assert torch.cuda.mem_get_info(cuda)[0] == free1, f"{what}: device memory allocated on call {call}"
    assert alloc1 >= alloc0 and free1 <= free0
