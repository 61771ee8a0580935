"""B200-native exact scaled-dot-product attention: tiled prefill, paged decode and the paged KV cache.

The compute path is libattn_b200.so (CUDA for sm_100a, C ABI in
include/attn_b200.h); ``api`` marshals torch tensors into it.  Importing the
package does not load the library; the first call does, and raises if the
library has not been built.
"""
from .api import (AttnError, PagePool, attn_decode_paged, attn_decode_paged_noalloc,  # noqa: F401
                  attn_decode_paged_fp8, attn_decode_paged_workspace_size, attn_kv_append,
                  attn_kv_append_fp8,
                  attn_device_status, attn_prefill, attn_prefill_f32, attn_prefill_f32_lse, attn_prefill_lse,
                  attn_prefill_host, attn_prefill_paged,
                  attn_status_string, attn_version)
