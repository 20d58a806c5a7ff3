"""B200-native Gated DeltaNet hot path (InfiniteVL's linear token mixer).

Chunkwise prefill with a carried fp32 state, a bandwidth-bound decode step and
the layer steps around them (short convolution / norms / gates before, the
output gate after), written as CUDA kernels for sm_100a behind the C ABI in
``include/gdn.h``.
This package is the thin Python binding of that library.
"""
from .gdn import (ACT_NONE, ACT_SILU, CHUNK, GATE_SIGMOID, GATE_SILU, GDN_BF16, GDN_F32, GdnError,
                  GdnSession, declared_symbols, gdn_decode_step, gdn_layer_prefill, gdn_layer_prefill_workspace_size,
                  gdn_output_gate, gdn_prefill, gdn_prefill_kernel_count,
                  gdn_noalloc_read_status, gdn_prefill_noalloc, gdn_prefill_workspace_size, gdn_preprocess,
                  gdn_read_status, gdn_rope, gdn_set_wait_limit, WAIT_LIMIT_DEFAULT,
                  gdn_swa_attention, library, status_string)

__all__ = ["ACT_NONE", "ACT_SILU", "CHUNK", "GATE_SIGMOID", "GATE_SILU", "GDN_BF16", "GDN_F32", "GdnError", "GdnSession",
           "declared_symbols", "gdn_decode_step", "gdn_layer_prefill", "gdn_layer_prefill_workspace_size",
           "gdn_output_gate", "gdn_prefill", "gdn_prefill_kernel_count",
           "gdn_noalloc_read_status", "gdn_prefill_noalloc", "gdn_prefill_workspace_size", "gdn_preprocess", "gdn_read_status", "gdn_rope", "gdn_set_wait_limit", "WAIT_LIMIT_DEFAULT", "gdn_swa_attention",
           "library", "status_string"]
