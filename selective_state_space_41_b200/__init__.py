"""libselscan: the Mamba selective-scan forward as hand-written sm_100a CUDA
kernels behind a C ABI (``include/selscan.h``), with a thin Python binding.

    from selective_state_space_41_b200 import selective_scan_fwd
    y, last = selective_scan_fwd(u, delta, A, B, C, D, z, delta_bias,
                                 delta_softplus=True, return_last_state=True)

``workloads`` and ``gen`` hold the synthetic workloads and their seeded input
generator.
"""
from .selscan import (SS_BF16, SS_F32, SelscanError, lib, selective_scan_bwd, selective_scan_fwd,  # noqa: F401
                      ss_bwd, ss_bwd_workspace_bytes, ss_fwd, ss_step,
                      ss_fwd_heuristic, ss_fwd_hostio, ss_fwd_noalloc, ss_fwd_workspace_bytes,
                      ss_status_string, ss_fwd_dtproj, ss_fwd_xdbl, ss_bwd_heuristic, ss_device_status,
                      ss_fwd_ckpt, ss_bwd_ckpt, ss_bwd_ckpt_workspace_bytes, ckpt_shape,
                      SelectiveScanFn, selective_scan_fn,
                      ss_version, workspace_for)

__all__ = ["selective_scan_fwd", "selective_scan_bwd", "ss_bwd", "ss_bwd_workspace_bytes", "ss_fwd", "ss_step", "ss_fwd_heuristic", "ss_fwd_hostio", "ss_fwd_noalloc",
           "ss_fwd_workspace_bytes", "workspace_for", "ss_status_string", "ss_version",
           "ss_fwd_dtproj", "ss_fwd_xdbl", "ss_bwd_heuristic", "ss_device_status",
           "ss_fwd_ckpt", "ss_bwd_ckpt", "ss_bwd_ckpt_workspace_bytes", "ckpt_shape",
           "SelectiveScanFn", "selective_scan_fn",
           "SelscanError", "SS_F32", "SS_BF16", "lib"]
