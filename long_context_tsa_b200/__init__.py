"""Token Sparse Attention prefill hot path on B200 (sm_100a).

The compute lives in ``libtsa.so`` (CUDA kernels behind the C ABI of
``include/tsa.h``); ``_native`` is its ctypes binding.  Importing this package
does not load the library; the first call does, and fails loudly if it is
missing.
"""

from ._native import (  # noqa: F401
    TSA_BF16,
    TSA_F32,
    TsaDesc,
    TsaError,
    alloc_drift_workspace,
    alloc_out_proj_workspace,
    alloc_workspace,
    desc_for,
    make_desc,
    tsa_attend,
    tsa_attend_accumulate,
    tsa_attend_block_sparse,
    tsa_check_status,
    tsa_debug_exp2,
    tsa_debug_launch_count,
    tsa_debug_cta_pair_launch_count,
    tsa_debug_set_wait_limit,
    tsa_debug_wait_never_set,
    tsa_drift,
    tsa_drift_workspace_size,
    tsa_forward,
    tsa_forward_coverage,
    tsa_forward_host,
    tsa_forward_host_h2d_bytes,
    tsa_layer_stable,
    tsa_out_proj,
    tsa_out_proj_workspace_size,
    tsa_score,
    tsa_score_noalloc,
    tsa_select,
    tsa_select_coverage,
    tsa_status_string,
    tsa_workspace_init,
    tsa_workspace_size,
    tsa_zero_dropped,
)
