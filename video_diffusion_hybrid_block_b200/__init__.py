"""B200 (sm_100a) forward pass of VideoDeltaNet's hybrid attention layer.

The compute lives in libvdn.so (C ABI, include/vdn.h); ``binding`` marshals
torch tensors into it; ``branch_parallel`` places the two branches on two
ranks.
"""
from .binding import (  # noqa: F401
    EXPORTED, LIB_PATH, PROFILE_GROUPS, VDN_BF16, VDN_F32, VDN_PROJ_BF16, VDN_PROJ_FP8, Shape,
    VdnError, alloc_fp8_workspace, alloc_proj_workspace, alloc_workspace, load_library,
    vdn_bsa_fwd, vdn_bsa_fwd_fp8, vdn_bsa_merge_fwd, vdn_error_string, vdn_fp8_workspace_bytes,
    vdn_gate_merge, vdn_get_device_error, vdn_hybrid_attn_branches, vdn_hybrid_attn_fwd,
    vdn_hybrid_attn_fwd_fp8, vdn_hybrid_attn_fwd_profile, vdn_hybrid_attn_proj_fwd, vdn_linear,
    vdn_pair_audit, vdn_proj_workspace_bytes, vdn_quantize_rows_e4m3, vdn_read_images_bytes,
    vdn_selftest_wait_timeout, vdn_vda_read_images, vdn_vda_scan, vdn_vda_scan_noalloc,
    vdn_workspace_bytes,
)
