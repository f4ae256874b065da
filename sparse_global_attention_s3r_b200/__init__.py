"""B200 (sm_100a) sparse global attention of Speed3R: a C-ABI CUDA library (libs3r.so,
include/s3r.h) and its thin torch binding.

    from sparse_global_attention_s3r_b200 import Config, sparse_attn_fwd
"""
from .api import (Config, HostPipeline, SparseAttention, SparseAttentionFunction, alloc_workspace,
                  bwd_workspace_bytes, cmp_attn_and_score, compress_kv, gate_combine,
                  read_device_status, sel_attn, sparse_attn_bwd, sparse_attn_fwd, topk_blocks,
                  workspace_bytes)

__all__ = ["Config", "HostPipeline", "SparseAttention", "SparseAttentionFunction",
           "alloc_workspace", "bwd_workspace_bytes", "cmp_attn_and_score", "compress_kv",
           "gate_combine", "read_device_status", "sel_attn", "sparse_attn_bwd", "sparse_attn_fwd",
           "topk_blocks", "workspace_bytes"]
