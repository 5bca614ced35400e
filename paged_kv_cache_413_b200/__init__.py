"""B200-native paged KV-cache decode (PagedAttention) for sm_100a.

The compute lives in ``libpa.so`` (hand-written CUDA kernels behind the C ABI in
``include/pa.h``); this package holds its thin ctypes binding (``binding``), the
build step (``build``) and the seeded synthetic workloads (``workloads``).
"""

from .binding import (PaError, library, library_path, pa_copy_blocks, pa_get_device_error,
                      pa_paged_attention_decode, pa_paged_attention_decode_shared_prefix,
                      pa_paged_attention_decode_static_workspace,
                      pa_paged_attention_partition_size, pa_paged_attention_prefill,
                      pa_paged_attention_workspace_size,
                      pa_reshape_and_cache, pa_status_string, pa_swap_blocks)

__all__ = ["PaError", "library", "library_path", "pa_copy_blocks", "pa_get_device_error",
           "pa_paged_attention_decode", "pa_paged_attention_decode_shared_prefix",
           "pa_paged_attention_decode_static_workspace",
           "pa_paged_attention_partition_size", "pa_paged_attention_prefill",
           "pa_paged_attention_workspace_size",
           "pa_reshape_and_cache", "pa_status_string", "pa_swap_blocks"]
