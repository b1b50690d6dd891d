"""SparsePR attention operator for NVIDIA B200 (sm_100a).

The operator (arXiv 2608.18484) runs Response-Coupled Partitioning, centroid block
routing, block-sparse attention and Probe-Fitted Residual Reconstruction in one call.
All arithmetic runs in the CUDA library libsparsepr.so behind the C ABI declared in
include/sparsepr.h; this package is its Python binding.
"""
from .sparsepr import (  # noqa: F401
    BF16, ERR_CUDA, ERR_INVALID_ARG, ERR_NONFINITE, ERR_TIMEOUT, ERR_UNSUPPORTED, EXPORTED_SYMBOLS, F32, OK,
    WEIGHT_INV_NORM, WEIGHT_UNIFORM, RIDGE_RELATIVE, PARTITION_RESPONSE, PARTITION_SEMANTIC, ROUTE_CENTROID, ROUTE_SIZE_CORRECTED, ROUTE_LSE,
    BUDGET_UNIFORM, BUDGET_GLOBAL,
    Partition, SparsePRConfig, SparsePRError, apply_residual, attention, check,
    dense_attn, fit_residual, fit_residual_noalloc, lib, new_workspace, num_groups, partition, probe_dense, probe_rows, route, route_k,
    sparse_attn, sparse_attn_apply, fused_supported, reset_workspace, attention_call, attention_host, call_workspace,
    host_workspace, test_fill, test_topk, test_partition_trace, load_library, workspace_size, row_errors, launch_count,
    kernel_timing, kernel_timing_read,
)
