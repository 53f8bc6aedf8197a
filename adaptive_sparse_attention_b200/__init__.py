"""B200-native (sm_100a) causal alpha-entmax attention with adaptive block skipping (forward
pass, and its backward pass on the CUDA cores), as a C-ABI library (libentmax_attn.so,
include/entmax_attn.h) with a thin torch binding.  The computation runs only in the library's
CUDA kernels."""
from .api import (alloc_outputs, alloc_workspace, decode_block_mask, entmax_attn_bwd,
                  entmax_attn_fwd, entmax_attn_fwd_host, entmax_attn_fwd_no_block_mask,
                  entmax_attn_fwd_noalloc,
                  entmax_rows, entmax_attn_fused, entmax_attn_screened, entmax_attn_two_pass,
                  fallback_tiles, mask_layout, mask_words,
                  out_pass, route_chunks, screen_bytes, status, tau_pass, tau_pass_screened, tile_slot_table, workspace_bytes,
                  workspace_min_bytes)

__all__ = ["entmax_attn_fwd", "entmax_attn_fwd_host", "entmax_attn_bwd", "entmax_attn_fwd_no_block_mask",
           "entmax_attn_fwd_noalloc", "entmax_attn_two_pass", "entmax_attn_fused",
           "entmax_attn_screened", "tau_pass_screened", "screen_bytes", "tau_pass",
           "out_pass",
           "alloc_outputs", "alloc_workspace", "workspace_bytes", "workspace_min_bytes",
           "mask_layout", "mask_words", "decode_block_mask", "tile_slot_table", "fallback_tiles",
           "status", "entmax_rows", "route_chunks"]
