"""Frame-wise Gated DeltaNet (GDN) forward pass for SANA-WM on B200 (sm_100a).

The compute lives in ``lib/libgdn.so`` (CUDA, C ABI declared in ``include/gdn.h``);
``gdn`` is its ctypes binding.
"""

from .gdn import (GATE_EVERY_TOKEN, GATE_FRAME_START, GDN_ERR_CUDA, GDN_ERR_INVALID_ARG, GDN_ERR_TIMEOUT,
                  GDN_ERR_UNSUPPORTED, GDN_OK, GdnError, bidir_workspace, forward, forward_bidirectional,
                  gdn_bf16_path, gdn_bidir_workspace_bytes, gdn_forward, gdn_forward_bidir, gdn_forward_bidir_f32, gdn_forward_fp8,
                  gdn_forward_f32, gdn_forward_gated, gdn_forward_gated_f32, gdn_forward_host, gdn_forward_host_ws,
                  gdn_forward_static_ws, gdn_forward_ws, gdn_get_last_device_status, gdn_set_wait_limit_ns,
                  gdn_softmax_attention, softmax_attention,
                  gdn_state_step, gdn_state_step_f32, gdn_state_step_ws, gdn_version, gdn_workspace_bytes, load,
                  state_step, status_string, workspace)

__all__ = ["GATE_EVERY_TOKEN", "GATE_FRAME_START", "GDN_OK", "GDN_ERR_INVALID_ARG", "GDN_ERR_UNSUPPORTED",
           "GDN_ERR_CUDA", "GDN_ERR_TIMEOUT", "GdnError", "forward", "forward_bidirectional", "state_step",
           "workspace", "bidir_workspace", "gdn_forward", "gdn_state_step", "gdn_forward_f32",
           "gdn_state_step_f32", "gdn_forward_host", "gdn_workspace_bytes", "gdn_forward_ws",
           "gdn_state_step_ws", "gdn_forward_host_ws", "gdn_forward_static_ws", "gdn_forward_gated",
           "gdn_forward_gated_f32", "gdn_bidir_workspace_bytes", "gdn_forward_bidir", "gdn_forward_bidir_f32", "gdn_forward_fp8",
           "gdn_softmax_attention", "softmax_attention", "gdn_get_last_device_status", "gdn_set_wait_limit_ns", "gdn_bf16_path", "gdn_version", "load",
           "status_string"]
