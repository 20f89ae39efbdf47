"""B200 (sm_100a) DeepSeek Sparse Attention forward: lightning indexer -> top-k selection -> sparse MLA.

The computation lives in libdsa.so (hand-written CUDA, C ABI in include/dsa.h); this package only builds it
(`build.py`) and binds it (`_lib.py`).  Importing the package loads the library and fails if it is missing.
"""
from ._lib import (  # noqa: F401
    DsaError,
    dsa_check_bounded_wait,
    dsa_decode_noalloc_scratch_bytes,
    dsa_decode_paged_workspace_size,
    dsa_decode_workspace_size,
    dsa_forward_decode_noalloc,
    dsa_forward_decode,
    dsa_forward_decode_paged,
    dsa_forward_prefill,
    dsa_forward_prefill_host,
    dsa_forward_prefill_kl,
    dsa_forward_prefill_rows,
    dsa_forward_prefill_varlen,
    dsa_get_device_status,
    dsa_indexer_kl,
    dsa_indexer_scores,
    dsa_launch_count,
    dsa_num_sms,
    dsa_prefill_block_rows,
    dsa_prefill_host_workspace_size,
    dsa_prefill_kl_workspace_size,
    dsa_prefill_rows_workspace_size,
    dsa_prefill_select,
    dsa_prefill_varlen_workspace_size,
    dsa_prefill_workspace_size,
    dsa_sparse_mla_attn,
    dsa_topk,
    prefill_blocks,
)
