"""B200-native Gated DeltaNet hot path (InfiniteVL's linear token mixer).

Chunkwise prefill with a carried fp32 state and a bandwidth-bound decode step,
written as CUDA kernels for sm_100a behind the C ABI in ``include/gdn.h``.
This package is the thin Python binding of that library.
"""
from .gdn import (CHUNK, GDN_BF16, GDN_F32, GdnError, declared_symbols, gdn_decode_step,
                  gdn_prefill, gdn_prefill_kernel_count, gdn_prefill_noalloc, gdn_prefill_workspace_size, library, status_string)

__all__ = ["CHUNK", "GDN_BF16", "GDN_F32", "GdnError", "declared_symbols", "gdn_decode_step",
           "gdn_prefill", "gdn_prefill_kernel_count", "gdn_prefill_noalloc", "gdn_prefill_workspace_size", "library", "status_string"]
