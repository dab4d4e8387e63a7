"""Helpers shared by the GPU tests: upload seeded inputs, run the library, compare
with the float64 oracle.  Parity bars (written in the tests that use them):
bf16 q/k/v/out with float32 state: max-abs <= 2e-2 and relative L2 <= 5e-3;
float32 reference mode: relative L2 <= 1e-4.  Both bars apply to `out` and to
the final state.
"""

import numpy as np

from workloads import bf16_bits

BF16_MAX_ABS = 2e-2
BF16_REL_L2 = 5e-3
F32_REL_L2 = 1e-4


def to_device(x, io_dtype, device):
    import torch
    if io_dtype == "bf16":
        t = torch.from_numpy(bf16_bits(x).view(np.int16).copy()).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(device)


def f32_device(x, device):
    import torch
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(device)


def upload(inp, device):
    """Device tensors q, k, v (io dtype), gate, beta (float32)."""
    return (to_device(inp.q, inp.io_dtype, device), to_device(inp.k, inp.io_dtype, device),
            to_device(inp.v, inp.io_dtype, device), f32_device(inp.gate, device),
            f32_device(inp.beta, device))


def host(t):
    return t.float().cpu().numpy().astype(np.float64)


def rel_l2(x, ref):
    x = np.asarray(x, np.float64); ref = np.asarray(ref, np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(x - ref) / (den if den > 0 else 1.0))


def max_abs(x, ref):
    return float(np.max(np.abs(np.asarray(x, np.float64) - np.asarray(ref, np.float64)))) if np.size(ref) else 0.0


def assert_bf16_parity(x, ref, what):
    e_abs, e_rel = max_abs(x, ref), rel_l2(x, ref)
    assert e_abs <= BF16_MAX_ABS and e_rel <= BF16_REL_L2, \
        f"{what}: max-abs {e_abs:.3e} (bar {BF16_MAX_ABS}), rel-L2 {e_rel:.3e} (bar {BF16_REL_L2})"
    return e_abs, e_rel


def assert_f32_parity(x, ref, what):
    e_rel = rel_l2(x, ref)
    assert e_rel <= F32_REL_L2, f"{what}: rel-L2 {e_rel:.3e} (bar {F32_REL_L2})"
    return e_rel


def run_library(inp, device, state_in=None, want_state=True, chunk_len=64, canary=True, ws=False):
    """Run gdn_forward (bf16; gdn_forward_ws with a fresh workspace if `ws`) or
    gdn_forward_f32 through the C ABI.

    Outputs are NaN-filled first and surrounded by guard bands filled with a
    sentinel; the guards must come back untouched and no NaN may remain.
    """
    import torch
    import hybrid_linear_attention_frame_b200 as G
    q, k, v, g, b = upload(inp, device)
    Bn, T, H, dk = inp.q.shape
    dv = inp.v.shape[3]
    dt = q.dtype
    guard = 64
    n_out = Bn * T * H * dv
    out_buf = torch.full((n_out + 2 * guard,), float("nan"), dtype=dt, device=device)
    out_buf[:guard] = 7.0
    out_buf[-guard:] = 7.0
    out = out_buf[guard:guard + n_out]
    n_st = Bn * H * dk * dv
    st_buf = torch.full((n_st + 2 * guard,), float("nan"), dtype=torch.float32, device=device)
    st_buf[:guard] = 7.0
    st_buf[-guard:] = 7.0
    st = st_buf[guard:guard + n_st] if want_state else None
    s_in = None if state_in is None else f32_device(state_in, device)
    if ws and inp.io_dtype == "bf16":
        wsp = G.workspace(Bn, H, T, dk, dv, chunk_len, device)
        if wsp is not None:
            wsp.fill_(0xA5)          # garbage: the call must not depend on its contents
        G.gdn_forward_ws(q, k, v, g, b, s_in, st, out, Bn, H, T, dk, dv, inp.frame_len, chunk_len,
                         wsp)
    else:
        fn = G.gdn_forward_f32 if inp.io_dtype == "f32" else G.gdn_forward
        fn(q, k, v, g, b, s_in, st, out, Bn, H, T, dk, dv, inp.frame_len, chunk_len)
    torch.cuda.synchronize()
    assert G.gdn_get_last_device_status() == G.GDN_OK
    if canary:
        assert bool((out_buf[:guard] == 7.0).all()) and bool((out_buf[-guard:] == 7.0).all()), \
            "write outside out"
        assert bool((st_buf[:guard] == 7.0).all()) and bool((st_buf[-guard:] == 7.0).all()), \
            "write outside state_out"
        assert not bool(torch.isnan(out).any()), "out not fully written"
        if want_state:
            assert not bool(torch.isnan(st).any()), "state_out not fully written"
    o = host(out).reshape(Bn, T, H, dv)
    s = host(st).reshape(Bn, H, dk, dv) if want_state else None
    return o, s
