"""B200 (sm_100a) decode-step hybrid sparse + linear attention.

The computation lives in ``libhyb_attn.so`` (hand-written CUDA kernels behind
the C ABI of ``include/hyb_attn.h``).  This package only marshals arguments
(``_abi``) and, in ``HybridAttentionLayer``, allocates the caller-owned device
buffers with PyTorch.
"""

from ._abi import (  # noqa: F401
    HybAttnError,
    hyb_attn_config,
    hyb_attn_buffers,
    hyb_attn_sizes,
    hyb_attn_plan_info,
    hyb_attn_query_sizes,
    hyb_attn_workspace_size,
    hyb_attn_plan,
    hyb_attn_init,
    hyb_attn_init_rows,
    hyb_attn_attach,
    hyb_attn_attach_rows,
    hyb_attn_append,
    hyb_attn_append_chunk,
    hyb_attn_sync_state,
    hyb_attn_decode,
    hyb_attn_decode_append,
    hyb_attn_decode_chunk,
    hyb_attn_decode_with_selection,
    hyb_attn_decode_strided,
    hyb_attn_step_host,
    hyb_attn_step_layers_staging_bytes,
    hyb_attn_step_layers_host,
    hyb_attn_decode_noalloc,
    hyb_attn_length,
    hyb_attn_row_length,
    hyb_attn_status,
    hyb_attn_set_timing_events,
    hyb_attn_set_wait_limit,
    hyb_attn_set_test_flags,
    hyb_attn_destroy,
    hyb_attn_strerror,
    hyb_attn_last_cuda_error,
    load_library,
    LIB_PATH,
    HYB_STATUS_NONFINITE,
    HYB_STATUS_DENOMINATOR,
    HYB_STATUS_BAD_SELECTION,
    HYB_STATUS_TIMEOUT,
    HYB_STATUS_NAN_SCORE,
    HYB_TEST_WITHHOLD_SCORES,
)
from .layer import HybridAttentionLayer, make_config  # noqa: F401
