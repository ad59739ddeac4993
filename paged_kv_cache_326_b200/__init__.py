"""B200-native paged decode attention: the C-ABI library libpagedattn.so
(kernels in csrc/), its Python binding, and seeded synthetic workloads.

Importing the package does not load the library; the first call does, and
fails loudly if it was not built.
"""
from .binding import (PA_OPT_DECODE_WARPS, PA_OPT_GQA_KERNEL, PA_OPT_PREFILL_KERNEL,
                      PA_OPT_FP8_KERNEL, PA_OPT_PREFIX_KEY_BITS, PA_OPT_WAIT_LIMIT_NS,
                      BlockManager, PagedAttnError, kv_cache_write, lib, pa_copy_blocks,
                      pa_decode_step, pa_decode_step_fp8, pa_kv_cache_write_fp8, pa_paged_attn_decode_fp8,
                      pa_prefill, pa_prefill_with_prefix, pa_paged_attn_decode_shared,
                      pa_paged_attn_decode_shared_workspace_size, split_shared_prefix,
                      pa_kv_cache_write, pa_paged_attn_decode_gqa,
                      pa_paged_attn_decode, pa_paged_attn_decode_workspace_size,
                      pa_set_option, pa_status_string, paged_attn_decode)

__all__ = ["PA_OPT_DECODE_WARPS", "PA_OPT_GQA_KERNEL", "PA_OPT_PREFILL_KERNEL",
           "PA_OPT_FP8_KERNEL", "PA_OPT_PREFIX_KEY_BITS", "PA_OPT_WAIT_LIMIT_NS", "BlockManager", "pa_copy_blocks", "pa_kv_cache_write_fp8",
           "pa_paged_attn_decode_fp8", "pa_prefill", "pa_prefill_with_prefix", "PagedAttnError", "kv_cache_write", "lib", "pa_decode_step", "pa_decode_step_fp8",
           "pa_kv_cache_write", "pa_paged_attn_decode_gqa",
           "pa_paged_attn_decode", "pa_paged_attn_decode_workspace_size", "pa_set_option",
           "pa_status_string", "paged_attn_decode", "pa_paged_attn_decode_shared",
           "pa_paged_attn_decode_shared_workspace_size", "split_shared_prefix"]
