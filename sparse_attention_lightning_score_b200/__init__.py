"""B200-native lightning-indexer scan (DSA) with LatentIndex extensions.

The hot path runs in ``libli.so`` (hand-written sm_100a CUDA behind the C ABI
in ``include/li.h``); ``api`` is its thin PyTorch binding and ``synth`` makes
the seeded synthetic inputs.
"""
from .api import (LiError, li_absorb_query, li_absorb_query_layers, li_copy_from_host,  # noqa: F401
                  li_decode_score_hist, li_decode_select, li_decode_select_finish, li_decode_select_score,
                  li_decode_select_workspace, li_get_last_error,
                  li_host_device_pointer, li_hs_refine, li_hs_refine_fp8, li_hs_refine_workspace, li_index_score, li_latent_score, li_latent_score_fp8,
                  li_latent_score_hist, li_merge_shards, li_quantize_query, li_selftest_wait_timeout,
                  li_sparse_attention, li_sparse_attention_workspace, li_topk, li_topk_hist)

__all__ = ["LiError", "li_absorb_query", "li_absorb_query_layers", "li_copy_from_host", "li_decode_score_hist",
           "li_decode_select", "li_decode_select_finish", "li_decode_select_score", "li_decode_select_workspace", "li_get_last_error", "li_host_device_pointer",
           "li_hs_refine", "li_hs_refine_fp8", "li_hs_refine_workspace", "li_index_score", "li_latent_score", "li_latent_score_fp8", "li_latent_score_hist",
           "li_merge_shards", "li_quantize_query", "li_selftest_wait_timeout", "li_sparse_attention",
           "li_sparse_attention_workspace", "li_topk", "li_topk_hist"]
