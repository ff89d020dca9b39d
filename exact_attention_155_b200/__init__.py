"""B200 (sm_100a) exact attention: fused forward with LSE, recompute backward and
KV-cache decode, exposed through the C ABI of libfa.so (include/fa.h).

The CUDA library is loaded lazily on the first call, so importing the package (for
example for its seeded input generators) needs no GPU. Calls raise if the library
is missing or the device is not sm_100.
"""
from .interface import (flash_attn_func, flash_attn_qkvpacked_func,  # noqa: F401
                        flash_attn_varlen_func, flash_attn_with_kvcache)
from .ops import (FAError, accumulate, bwd, bwd_ex, bwd_qkvpacked, bwd_workspace_size,  # noqa: F401
                  decode, decode_paged, decode_workspace_size, device_status, fwd, fwd_ex,
                  fwd_qkvpacked, load_library, merge_partials)

__all__ = ["FAError", "fwd", "bwd", "fwd_ex", "bwd_ex", "fwd_qkvpacked", "bwd_qkvpacked", "decode",
           "decode_paged", "merge_partials", "accumulate",
           "bwd_workspace_size", "decode_workspace_size", "device_status", "load_library",
           "flash_attn_func", "flash_attn_qkvpacked_func", "flash_attn_varlen_func",
           "flash_attn_with_kvcache"]
