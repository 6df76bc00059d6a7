"""Selection-driven block-sparse causal attention for NVIDIA B200 (sm_100a).

The CUDA kernels sit behind the C-ABI library ``libspa.so`` (``include/spa.h``);
:mod:`block_sparse_long_stats_b200.spa` is its thin Python binding. Build with
``python -m block_sparse_long_stats_b200.build``.
"""
from .spa import (SpaError, decode, lib, prefill, spa_block_stats, spa_decode_workspace_bytes,
                  spa_get_device_error, spa_last_error, spa_quantize_block_stats,
                  spa_quantized_stats_bytes, spa_rla_block_states, spa_rla_decode_state,
                  spa_rla_decode_workspace_bytes, spa_rla_prefill, spa_select_quantized,
                  spa_select_score_order, spa_sparse_attn_prefill_early_stop, spa_block_stats_quantized,
                  spa_pbs_gather, spa_pbs_permutation, spa_pbs_workspace_bytes,
                  spa_select_segperm, spa_prefill_host, spa_prefill_host_workspace_bytes,
                  spa_selftest_wait_timeout, spa_sparse_attn_prefill_segperm,
                  spa_sparse_attn_decode_rla,
                  spa_select, spa_sparse_attn_decode, spa_sparse_attn_prefill, spa_status_string)

__all__ = ["SpaError", "decode", "lib", "prefill", "spa_block_stats",
           "spa_decode_workspace_bytes", "spa_get_device_error", "spa_last_error",
           "spa_quantize_block_stats", "spa_quantized_stats_bytes", "spa_select_quantized",
           "spa_select_score_order", "spa_sparse_attn_prefill_early_stop", "spa_block_stats_quantized",
           "spa_pbs_gather", "spa_pbs_permutation", "spa_pbs_workspace_bytes", "spa_select_segperm",
           "spa_prefill_host", "spa_prefill_host_workspace_bytes", "spa_selftest_wait_timeout",
           "spa_sparse_attn_prefill_segperm",
           "spa_rla_block_states", "spa_rla_decode_state", "spa_rla_decode_workspace_bytes",
           "spa_rla_prefill", "spa_select", "spa_sparse_attn_decode_rla",
           "spa_sparse_attn_decode", "spa_sparse_attn_prefill", "spa_status_string"]
