"""Python binding of libgdn.so: argument marshalling only.

Every function here has the name and argument order of the C entry point in
``include/gdn.h``.  Tensors are passed as raw device pointers (``data_ptr()``)
and the stream defaults to PyTorch's current stream; all arithmetic happens in
the library's CUDA kernels.  If the library cannot be loaded the import fails
loudly; there is no fallback implementation.
"""

import ctypes
import os
from typing import Optional

from . import build as _build

GDN_OK = 0
GDN_ERR_INVALID_ARG = -1
GDN_ERR_UNSUPPORTED = -2
GDN_ERR_CUDA = -3
GDN_ERR_TIMEOUT = -4

EXPORTS = ("gdn_forward", "gdn_state_step", "gdn_forward_f32", "gdn_state_step_f32",
           "gdn_forward_host", "gdn_workspace_bytes", "gdn_forward_ws", "gdn_state_step_ws",
           "gdn_forward_host_ws", "gdn_forward_static_ws", "gdn_forward_gated",
           "gdn_forward_gated_f32", "gdn_bidir_workspace_bytes", "gdn_forward_bidir",
           "gdn_forward_bidir_f32", "gdn_forward_fp8", "gdn_softmax_attention", "gdn_set_wait_limit_ns", "gdn_status_string",
           "gdn_get_last_device_status", "gdn_bf16_path", "gdn_version")


class GdnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


_lib = None


def library_path() -> str:
    return _build.LIB_PATH


def load(build_if_missing: bool = True) -> ctypes.CDLL:
    """Load libgdn.so (building it first if it is missing and nvcc is available)."""
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if not os.path.exists(path):
        if not build_if_missing:
            raise OSError(f"libgdn.so not found at {path}; run "
                          "`python -m hybrid_linear_attention_frame_b200.build`")
        _build.build()
    lib = ctypes.CDLL(path)
    P, I = ctypes.c_void_p, ctypes.c_int
    fwd = [P] * 8 + [I] * 7 + [P]
    step = [P] * 7 + [I] * 7 + [P]
    for name, args in (("gdn_forward", fwd), ("gdn_forward_f32", fwd),
                       ("gdn_state_step", step), ("gdn_state_step_f32", step)):
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = I
    lib.gdn_forward_host.argtypes = [P] * 15 + [I] * 7 + [P]
    lib.gdn_forward_host.restype = I
    Z = ctypes.c_size_t
    lib.gdn_workspace_bytes.argtypes = [I] * 6 + [ctypes.POINTER(Z)]
    lib.gdn_workspace_bytes.restype = I
    lib.gdn_forward_ws.argtypes = [P] * 8 + [I] * 7 + [P, Z, P]
    lib.gdn_forward_ws.restype = I
    lib.gdn_state_step_ws.argtypes = [P] * 7 + [I] * 7 + [P, Z, P]
    lib.gdn_state_step_ws.restype = I
    lib.gdn_forward_host_ws.argtypes = [P] * 15 + [I] * 7 + [P, Z, P]
    lib.gdn_forward_host_ws.restype = I
    lib.gdn_forward_static_ws.argtypes = fwd
    lib.gdn_forward_static_ws.restype = I
    lib.gdn_forward_gated.argtypes = [P] * 8 + [I] * 8 + [P, Z, P]
    lib.gdn_forward_gated.restype = I
    lib.gdn_forward_gated_f32.argtypes = [P] * 8 + [I] * 8 + [P]
    lib.gdn_forward_gated_f32.restype = I
    lib.gdn_bidir_workspace_bytes.argtypes = [I] * 7 + [ctypes.POINTER(Z)]
    lib.gdn_bidir_workspace_bytes.restype = I
    lib.gdn_forward_bidir.argtypes = [P] * 6 + [I] * 7 + [P, Z, P]
    lib.gdn_forward_bidir.restype = I
    lib.gdn_forward_bidir_f32.argtypes = [P] * 6 + [I] * 7 + [P, Z, P]
    lib.gdn_forward_bidir_f32.restype = I
    lib.gdn_forward_fp8.argtypes = [P] * 3 + [ctypes.c_float] + [P] * 5 + [I] * 7 + [P]
    lib.gdn_forward_fp8.restype = I
    lib.gdn_softmax_attention.argtypes = [P] * 4 + [I] * 9 + [P]
    lib.gdn_softmax_attention.restype = I
    lib.gdn_status_string.argtypes = [I]
    lib.gdn_status_string.restype = ctypes.c_char_p
    lib.gdn_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong]
    lib.gdn_set_wait_limit_ns.restype = I
    lib.gdn_get_last_device_status.argtypes = [P]
    lib.gdn_get_last_device_status.restype = I
    lib.gdn_bf16_path.argtypes = [I, I, I]
    lib.gdn_bf16_path.restype = I
    lib.gdn_version.argtypes = []
    lib.gdn_version.restype = I
    _lib = lib
    return lib


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def status_string(status: int) -> str:
    return load().gdn_status_string(int(status)).decode()


def _check(status: int, where: str, check: bool) -> int:
    if check and status != GDN_OK:
        raise GdnError(status, where)
    return status


def gdn_forward(q, k, v, gate_logit, beta_logit, state_in, state_out, out,
                B, H, T, d_k, d_v, frame_len, chunk_len, stream=None, check=True) -> int:
    st = load().gdn_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(gate_logit), _ptr(beta_logit),
                            _ptr(state_in), _ptr(state_out), _ptr(out),
                            B, H, T, d_k, d_v, frame_len, chunk_len, _stream(stream))
    return _check(st, "gdn_forward", check)


def gdn_forward_fp8(q8, k8, v8, v_scale, gate_logit, beta_logit, state_in, state_out, out,
                    B, H, T, d_k, d_v, frame_len, chunk_len, stream=None, check=True) -> int:
    """q8, k8, v8: e4m3 bytes (uint8 tensors); v = v_scale * e4m3(v8); out bf16."""
    st = load().gdn_forward_fp8(_ptr(q8), _ptr(k8), _ptr(v8), float(v_scale), _ptr(gate_logit),
                                _ptr(beta_logit), _ptr(state_in), _ptr(state_out), _ptr(out),
                                B, H, T, d_k, d_v, frame_len, chunk_len, _stream(stream))
    return _check(st, "gdn_forward_fp8", check)


def gdn_state_step(q, k, v, gate_logit, beta_logit, state, out,
                   B, H, T, d_k, d_v, frame_len, chunk_len, stream=None, check=True) -> int:
    st = load().gdn_state_step(_ptr(q), _ptr(k), _ptr(v), _ptr(gate_logit), _ptr(beta_logit),
                               _ptr(state), _ptr(out), B, H, T, d_k, d_v, frame_len, chunk_len,
                               _stream(stream))
    return _check(st, "gdn_state_step", check)


def gdn_forward_f32(q, k, v, gate_logit, beta_logit, state_in, state_out, out,
                    B, H, T, d_k, d_v, frame_len, chunk_len, stream=None, check=True) -> int:
    st = load().gdn_forward_f32(_ptr(q), _ptr(k), _ptr(v), _ptr(gate_logit), _ptr(beta_logit),
                                _ptr(state_in), _ptr(state_out), _ptr(out),
                                B, H, T, d_k, d_v, frame_len, chunk_len, _stream(stream))
    return _check(st, "gdn_forward_f32", check)


def gdn_state_step_f32(q, k, v, gate_logit, beta_logit, state, out,
                       B, H, T, d_k, d_v, frame_len, chunk_len, stream=None, check=True) -> int:
    st = load().gdn_state_step_f32(_ptr(q), _ptr(k), _ptr(v), _ptr(gate_logit), _ptr(beta_logit),
                                   _ptr(state), _ptr(out), B, H, T, d_k, d_v, frame_len,
                                   chunk_len, _stream(stream))
    return _check(st, "gdn_state_step_f32", check)


def gdn_forward_host(h_q, h_k, h_v, h_gate_logit, h_beta_logit, h_state_in, h_state_out, h_out,
                     d_q, d_k, d_v, d_gate_logit, d_beta_logit, d_state, d_out,
                     B, H, T, d_k_dim, d_v_dim, frame_len, chunk_len, stream=None,
                     check=True) -> int:
    st = load().gdn_forward_host(
        _ptr(h_q), _ptr(h_k), _ptr(h_v), _ptr(h_gate_logit), _ptr(h_beta_logit),
        _ptr(h_state_in), _ptr(h_state_out), _ptr(h_out),
        _ptr(d_q), _ptr(d_k), _ptr(d_v), _ptr(d_gate_logit), _ptr(d_beta_logit),
        _ptr(d_state), _ptr(d_out), B, H, T, d_k_dim, d_v_dim, frame_len, chunk_len,
        _stream(stream))
    return _check(st, "gdn_forward_host", check)


def gdn_workspace_bytes(B, H, T, d_k, d_v, chunk_len) -> int:
    n = ctypes.c_size_t(0)
    st = load().gdn_workspace_bytes(B, H, T, d_k, d_v, chunk_len, ctypes.byref(n))
    _check(st, "gdn_workspace_bytes", True)
    return int(n.value)


def _nbytes(ws) -> int:
    return 0 if ws is None else ws.numel() * ws.element_size()


def gdn_forward_ws(q, k, v, gate_logit, beta_logit, state_in, state_out, out,
                   B, H, T, d_k, d_v, frame_len, chunk_len, workspace, workspace_bytes=None,
                   stream=None, check=True) -> int:
    wb = _nbytes(workspace) if workspace_bytes is None else workspace_bytes
    st = load().gdn_forward_ws(_ptr(q), _ptr(k), _ptr(v), _ptr(gate_logit), _ptr(beta_logit),
                               _ptr(state_in), _ptr(state_out), _ptr(out),
                               B, H, T, d_k, d_v, frame_len, chunk_len, _ptr(workspace), wb,
                               _stream(stream))
    return _check(st, "gdn_forward_ws", check)


def gdn_state_step_ws(q, k, v, gate_logit, beta_logit, state, out,
                      B, H, T, d_k, d_v, frame_len, chunk_len, workspace, workspace_bytes=None,
                      stream=None, check=True) -> int:
    wb = _nbytes(workspace) if workspace_bytes is None else workspace_bytes
    st = load().gdn_state_step_ws(_ptr(q), _ptr(k), _ptr(v), _ptr(gate_logit), _ptr(beta_logit),
                                  _ptr(state), _ptr(out), B, H, T, d_k, d_v, frame_len, chunk_len,
                                  _ptr(workspace), wb, _stream(stream))
    return _check(st, "gdn_state_step_ws", check)


def gdn_forward_host_ws(h_q, h_k, h_v, h_gate_logit, h_beta_logit, h_state_in, h_state_out, h_out,
                        d_q, d_k, d_v, d_gate_logit, d_beta_logit, d_state, d_out,
                        B, H, T, d_k_dim, d_v_dim, frame_len, chunk_len, workspace,
                        workspace_bytes=None, stream=None, check=True) -> int:
    wb = _nbytes(workspace) if workspace_bytes is None else workspace_bytes
    st = load().gdn_forward_host_ws(
        _ptr(h_q), _ptr(h_k), _ptr(h_v), _ptr(h_gate_logit), _ptr(h_beta_logit),
        _ptr(h_state_in), _ptr(h_state_out), _ptr(h_out),
        _ptr(d_q), _ptr(d_k), _ptr(d_v), _ptr(d_gate_logit), _ptr(d_beta_logit),
        _ptr(d_state), _ptr(d_out), B, H, T, d_k_dim, d_v_dim, frame_len, chunk_len,
        _ptr(workspace), wb, _stream(stream))
    return _check(st, "gdn_forward_host_ws", check)


def gdn_forward_static_ws(q, k, v, gate_logit, beta_logit, state_in, state_out, out,
                          B, H, T, d_k, d_v, frame_len, chunk_len, stream=None, check=True) -> int:
    st = load().gdn_forward_static_ws(_ptr(q), _ptr(k), _ptr(v), _ptr(gate_logit), _ptr(beta_logit),
                                      _ptr(state_in), _ptr(state_out), _ptr(out),
                                      B, H, T, d_k, d_v, frame_len, chunk_len, _stream(stream))
    return _check(st, "gdn_forward_static_ws", check)


GATE_EVERY_TOKEN = 0
GATE_FRAME_START = 1


def gdn_forward_gated(q, k, v, gate_logit, beta_logit, state_in, state_out, out,
                      B, H, T, d_k, d_v, frame_len, chunk_len, gate_mode, workspace=None,
                      workspace_bytes=None, stream=None, check=True) -> int:
    wb = _nbytes(workspace) if workspace_bytes is None else workspace_bytes
    st = load().gdn_forward_gated(_ptr(q), _ptr(k), _ptr(v), _ptr(gate_logit), _ptr(beta_logit),
                                  _ptr(state_in), _ptr(state_out), _ptr(out),
                                  B, H, T, d_k, d_v, frame_len, chunk_len, gate_mode,
                                  _ptr(workspace), wb, _stream(stream))
    return _check(st, "gdn_forward_gated", check)


def gdn_forward_gated_f32(q, k, v, gate_logit, beta_logit, state_in, state_out, out,
                          B, H, T, d_k, d_v, frame_len, chunk_len, gate_mode, stream=None,
                          check=True) -> int:
    st = load().gdn_forward_gated_f32(_ptr(q), _ptr(k), _ptr(v), _ptr(gate_logit), _ptr(beta_logit),
                                      _ptr(state_in), _ptr(state_out), _ptr(out),
                                      B, H, T, d_k, d_v, frame_len, chunk_len, gate_mode,
                                      _stream(stream))
    return _check(st, "gdn_forward_gated_f32", check)


def gdn_bidir_workspace_bytes(B, H, T, d_k, d_v, chunk_len, elem_bytes=2) -> int:
    n = ctypes.c_size_t(0)
    st = load().gdn_bidir_workspace_bytes(B, H, T, d_k, d_v, chunk_len, elem_bytes, ctypes.byref(n))
    _check(st, "gdn_bidir_workspace_bytes", True)
    return int(n.value)


def gdn_forward_bidir(q, k, v, gate_logit, beta_logit, out, B, H, T, d_k, d_v, frame_len, chunk_len,
                      workspace, workspace_bytes=None, stream=None, check=True) -> int:
    wb = _nbytes(workspace) if workspace_bytes is None else workspace_bytes
    st = load().gdn_forward_bidir(_ptr(q), _ptr(k), _ptr(v), _ptr(gate_logit), _ptr(beta_logit), _ptr(out),
                                  B, H, T, d_k, d_v, frame_len, chunk_len, _ptr(workspace), wb,
                                  _stream(stream))
    return _check(st, "gdn_forward_bidir", check)


def gdn_forward_bidir_f32(q, k, v, gate_logit, beta_logit, out, B, H, T, d_k, d_v, frame_len, chunk_len,
                          workspace, workspace_bytes=None, stream=None, check=True) -> int:
    wb = _nbytes(workspace) if workspace_bytes is None else workspace_bytes
    st = load().gdn_forward_bidir_f32(_ptr(q), _ptr(k), _ptr(v), _ptr(gate_logit), _ptr(beta_logit),
                                      _ptr(out), B, H, T, d_k, d_v, frame_len, chunk_len, _ptr(workspace),
                                      wb, _stream(stream))
    return _check(st, "gdn_forward_bidir_f32", check)


def gdn_softmax_attention(q, k, v, out, B, H, T, d_k, d_v, frame_len, frames_per_block=3, cached_blocks=2,
                          sink_frames=1, stream=None, check=True) -> int:
    st = load().gdn_softmax_attention(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, T, d_k, d_v, frame_len,
                                      frames_per_block, cached_blocks, sink_frames, _stream(stream))
    return _check(st, "gdn_softmax_attention", check)


def gdn_set_wait_limit_ns(ns: int) -> int:
    return load().gdn_set_wait_limit_ns(int(ns))


def gdn_get_last_device_status(stream=None) -> int:
    return load().gdn_get_last_device_status(_stream(stream))


def gdn_bf16_path(d_k: int, d_v: int, chunk_len: int) -> int:
    return load().gdn_bf16_path(d_k, d_v, chunk_len)


def gdn_version() -> int:
    return load().gdn_version()


# ----------------------------------------------------------------------------
# tensor-level convenience wrappers (allocation by PyTorch, compute in the library)
# ----------------------------------------------------------------------------

def workspace(B, H, T, d_k, d_v, chunk_len=64, device="cuda"):
    """A workspace tensor for the *_ws calls (None if these sizes need none)."""
    import torch
    n = gdn_workspace_bytes(B, H, T, d_k, d_v, chunk_len)
    if n == 0:
        return None
    return torch.empty(n, dtype=torch.uint8, device=device)


def bidir_workspace(B, H, T, d_k, d_v, chunk_len=64, device="cuda", elem_bytes=2):
    """A workspace tensor for gdn_forward_bidir(_f32) (None when T = 0)."""
    import torch
    n = gdn_bidir_workspace_bytes(B, H, T, d_k, d_v, chunk_len, elem_bytes)
    if n == 0:
        return None
    return torch.empty(n, dtype=torch.uint8, device=device)


def forward_bidirectional(q, k, v, gate_logit, beta_logit, frame_len=880, chunk_len=64, stream=None, ws=None):
    """out = forward scan + backward scan (zero states) for bf16 or float32 q/k/v;
    ``ws`` from bidir_workspace, allocated here when not given."""
    import torch
    B, T, H, dk = q.shape
    dv = v.shape[3]
    f32 = q.dtype == torch.float32
    if ws is None:
        ws = bidir_workspace(B, H, T, dk, dv, chunk_len, q.device, 4 if f32 else 2)
    out = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    fn = gdn_forward_bidir_f32 if f32 else gdn_forward_bidir
    fn(q, k, v, gate_logit, beta_logit, out, B, H, T, dk, dv, frame_len, chunk_len, ws, stream=stream)
    return out


def softmax_attention(q, k, v, frame_len=880, frames_per_block=3, cached_blocks=2, sink_frames=1, stream=None):
    """out [B,T,H,d_v] = chunk-causal softmax attention of bf16 q, k [B,T,H,d_k], v [B,T,H,d_v]."""
    import torch
    B, T, H, dk = q.shape
    dv = v.shape[3]
    out = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    gdn_softmax_attention(q, k, v, out, B, H, T, dk, dv, frame_len, frames_per_block, cached_blocks, sink_frames,
                          stream)
    return out


def forward(q, k, v, gate_logit, beta_logit, state_in=None, frame_len=880, chunk_len=64,
            want_state=True, stream=None, ws=None):
    """out, state_out = forward(q [B,T,H,dk], k, v [B,T,H,dv], gate [B,F,H], beta [B,T,H], ...).

    bf16 q/k/v call gdn_forward (gdn_forward_ws when a workspace ``ws`` is
    given), float32 q/k/v call gdn_forward_f32.
    """
    import torch
    B, T, H, dk = q.shape
    dv = v.shape[3]
    out = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    st = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device) if want_state else None
    if q.dtype == torch.float32:
        gdn_forward_f32(q, k, v, gate_logit, beta_logit, state_in, st, out, B, H, T, dk, dv,
                        frame_len, chunk_len, stream)
    elif ws is not None:
        gdn_forward_ws(q, k, v, gate_logit, beta_logit, state_in, st, out, B, H, T, dk, dv,
                       frame_len, chunk_len, ws, stream=stream)
    else:
        gdn_forward(q, k, v, gate_logit, beta_logit, state_in, st, out, B, H, T, dk, dv,
                    frame_len, chunk_len, stream)
    return out, st


def state_step(q, k, v, gate_logit, beta_logit, state, frame_len=880, chunk_len=64,
               want_out=True, stream=None, ws=None):
    """Advance ``state`` in place over one streaming block; returns out (or None)."""
    import torch
    B, T, H, dk = q.shape
    dv = v.shape[3]
    out = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device) if want_out else None
    if q.dtype == torch.float32:
        gdn_state_step_f32(q, k, v, gate_logit, beta_logit, state, out, B, H, T, dk, dv,
                           frame_len, chunk_len, stream)
    elif ws is not None:
        gdn_state_step_ws(q, k, v, gate_logit, beta_logit, state, out, B, H, T, dk, dv,
                          frame_len, chunk_len, ws, stream=stream)
    else:
        gdn_state_step(q, k, v, gate_logit, beta_logit, state, out, B, H, T, dk, dv,
                       frame_len, chunk_len, stream)
    return out
