"""B200 (sm_100a) CSA / HCA attention hot path: thin Python binding of libcsa_b200.

Every function here only marshals arguments (torch tensors -> raw pointers and
sizes) and calls the C ABI declared in include/csa.h; all arithmetic runs in the
library's CUDA kernels.  There is no CPU fallback: loading fails loudly when the
shared library is missing, and calls raise on any non-zero status.
"""
from ._native import (  # noqa: F401
    CSA_BF16, CSA_F32, CSA_IFMT_E4M3, CSA_IFMT_F32, CSA_IFMT_MXFP4, CsaError, attn_decode_workspace_size, attn_merge_shards,
    csa_compress, csa_compress_kv8, grouped_out_proj, grouped_out_proj_workspace_size, hca_attn_decode, hca_attn_decode_kv8, hca_compress, hca_compress_attn_decode, index_key_compress, lib, lib_path, lightning_index, lightning_index_bf16, lightning_index_workspace_size, lightning_index_workspace_size_exact,
    launch_count, read_device_error, sparse_attn_decode, sparse_attn_decode_kv8, sparse_attn_decode_noalloc, sparse_attn_prefill, shard_topk_merge, topk_select,
    wait_probe, csa_decode_append, window_append, tensor_peak_probe,
)
