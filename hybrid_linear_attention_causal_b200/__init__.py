"""B200 (sm_100a) Gated DeltaNet layer: extend / decode / verify / commit behind a C ABI,
and the Mamba2 SSD chunk scan (ssd_combined_fwd).

The compute lives in libgdn.so (csrc/, declared in include/gdn.h and include/ssd.h); this
package holds its ctypes binding, the in-tree build step and seeded synthetic
workloads.  Calls fail loudly when libgdn.so has not been built.
"""
from .binding import (  # noqa: F401
    GDN_DEVERR_ACCEPT_RANGE,
    GDN_DEVERR_CKPT_RANGE,
    GDN_DEVERR_FP16_RANGE,
    GDN_DEVERR_SEQLENS,
    GDN_DEVERR_SLOT_RANGE,
    GDN_DEVERR_TIMEOUT,
    GDN_DEVERR_TREE,
    GDN_ERR_CUDA,
    GDN_ERR_INVALID_ARG,
    GDN_ERR_UNSUPPORTED,
    GDN_ERR_WORKSPACE,
    GDN_OK,
    GdnConfig,
    GdnError,
    SsdConfig,
    ssd_combined_fwd,
    ssd_workspace_size,
    alloc_workspace,
    gdn_commit,
    gdn_check_bounded_wait,
    gdn_commit_workspace_size,
    gdn_decode,
    gdn_decode_workspace_size,
    gdn_extend,
    gdn_extend_checkpoints,
    gdn_extend_static_scratch,
    gdn_extend_workspace_size,
    gdn_get_device_error,
    gdn_reset_device_error,
    gdn_set_launch_events,
    gdn_verify,
    gdn_verify_tree,
    gdn_verify_workspace_size,
)
