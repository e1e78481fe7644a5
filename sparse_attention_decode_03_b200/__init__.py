"""QSA (Qwen Sparse Attention) decode hot path for one NVIDIA B200 (sm_100a).

The compute runs in libqsa.so (hand-written CUDA, C ABI in include/qsa.h); this
package is its thin ctypes binding.  Build the library with
``python sparse_attention_decode_03_b200/build.py``.
"""
from .qsa import (  # noqa: F401
    ABI_VERSION, KV_BF16, KV_FP8_E4M3, LIB_PATH, BoundCall, Decoder, bind_append_kv, PagedCache, QSAError, StepGraph, StepIO, StepPipeline, dev_status_names, qsa_append_kv, qsa_combine,
    qsa_combine_f32, qsa_combine_ranks, qsa_dcp_localize_selection, qsa_dcp_localize_tokens, qsa_decode_plan, qsa_index_scores, qsa_index_topk, index_topk_smem_bytes, index_topk_resident_queries, fused_selection_pays, qsa_sparse_attention, qsa_sparse_attention_noalloc, qsa_sparse_decode, qsa_topk_blocks, splits_bound, status_string)
from .dcp import DCPRank, DCPShard  # noqa: F401,E402
