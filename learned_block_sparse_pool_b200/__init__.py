"""Veda-style learned block-sparse attention for video diffusion transformers,
B200-native (sm_100a): tile-pool + selector projection, fixed-budget top-k
tile selection, and block-sparse attention over the kept tiles plus dense
text / VLM / audio keys.

The computation lives in libveda.so (C ABI: include/veda.h); `binding` is a
ctypes marshalling layer over it.  Build the library with
`python -m learned_block_sparse_pool_b200.build`.
"""
from .binding import (EXPORTS, LIB_PATH, Problem, Selector, VedaError, alloc_indices, alloc_output, attn, attn_host, attn_host_buffer, dense_query_attn,
                      block_sparse_attn, check_status, fallback_rows, lib, pool_project, score_tiles, score_topk_tiles,
                      select_tiles,
                      select_tiles_noalloc, status_string, topk_tiles, workspace, workspace_size, workspace_view)

__all__ = ["EXPORTS", "LIB_PATH", "Problem", "Selector", "VedaError", "alloc_indices", "alloc_output", "attn", "attn_host", "attn_host_buffer", "dense_query_attn",
           "block_sparse_attn", "check_status", "fallback_rows", "lib", "pool_project", "score_tiles",
           "score_topk_tiles", "select_tiles",
           "select_tiles_noalloc", "status_string", "topk_tiles", "workspace", "workspace_size", "workspace_view"]
