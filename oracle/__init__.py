"""CPU oracle for paged decode attention (fp64 NumPy) and a reference model of
the block manager.

TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.  Only ``tests/``, the smoke
check in ``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may
import, call or run anything in this folder.  It shares no code with the CUDA
path and never imports the product package.
"""
from .paged_attention import (attend, cache_write, copy_blocks, decode_step, gather_context,
                              kv_head_of, paged_decode, paged_decode_shared, prefill,
                              prefill_with_prefix, split_shared_prefix)
from .block_manager import BlockManagerError, BlockManagerModel
from .fp8 import (cache_write_fp8, e4m3_decode, e4m3_encode, e4m3_value, paged_decode_fp8,
                  quantize)

__all__ = ["attend", "cache_write", "copy_blocks", "decode_step", "gather_context", "kv_head_of",
           "paged_decode", "prefill", "prefill_with_prefix",
           "paged_decode_shared", "split_shared_prefix",
           "BlockManagerError", "BlockManagerModel", "cache_write_fp8", "e4m3_decode",
           "e4m3_encode", "e4m3_value", "paged_decode_fp8", "quantize"]
