"""B200-native (sm_100a) attention forward with paged KV, GQA, varlen, causal/patch masks and fp8.

The compute path is the CUDA library libattn_b200.so (C ABI in include/attn_b200.h);
``binding`` marshals torch tensors into it.  ``workloads`` builds the seeded
synthetic inputs.
"""
from .binding import (AttnError, attn_check_device, attn_decode_paged,  # noqa: F401
                      attn_decode_workspace_size, attn_device_error, attn_fwd_dense,
                      attn_fwd_varlen_paged, MASK_CAUSAL, MASK_NONE, MASK_PATCH)
