"""B200 (sm_100a) packed causal attention with sequence-aware chunking.

Python binding of libsap.so (C ABI declared in include/sap.h).  Every step of
the computation runs in the library's CUDA kernels; this package only
marshals arguments (tensor pointers, sizes, the current CUDA stream) and owns
the plan handle.  PyTorch supplies device memory and streams.  There is no
fallback: if libsap.so is missing, importing a compute entry point raises.
"""
from ._capi import (  # noqa: F401
    SAP_TAG_CAUSAL,
    SAP_TAG_FULL,
    SAP_TAG_MASKED,
    SAP_WS_BWD,
    SAP_WS_FWD,
    Plan,
    SapError,
    alloc_workspace,
    library_path,
    load_library,
    sap_attn_bwd,
    sap_attn_bwd_kv_add,
    sap_attn_fwd,
    sap_attn_fwd_part,
    sap_attn_fwd_static_scratch,
    sap_device_status,
    sap_error_string,
    sap_balanced_chunks,
    sap_merge,
    sap_plan,
    sap_plan_bwd_direct,
    sap_plan_bwd_schedule,
    sap_plan_chunk_bounds,
    sap_plan_chunk_stats,
    sap_plan_chunks,
    sap_plan_fwd_local_units,
    sap_plan_destroy,
    sap_plan_fwd_schedule,
    sap_plan_items,
    sap_plan_rank,
    sap_plan_rank_spans,
    sap_plan_set_fused_merge,
    sap_plan_stats,
    sap_plan_upload,
    sap_plan_window,
    sap_set_forward_variant,
    sap_set_wait_limit_ns,
    sap_workspace_kv_offsets,
    sap_workspace_size,
)
