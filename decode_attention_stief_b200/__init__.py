"""B200 (sm_100a) StiefAttention latent-KV decode: Python binding of libstief.so.

The compute path is the CUDA library ``libstief.so`` (C ABI in include/stief.h).
This package only marshals torch tensors (device pointers, sizes, the current
stream) into those calls.  There is no CPU fallback: if the library cannot be
loaded, every call raises.
"""
from ._binding import (  # noqa: F401
    Prepared,
    StiefError,
    STATUS,
    DEV_CAPACITY_OVERFLOW,
    DEV_WAIT_TIMEOUT,
    DEV_BAD_LENGTH,
    library,
    library_path,
    prepare,
    stief_append_decode,
    stief_append_decode_paged,
    stief_compress_append,
    stief_compress_append_q8,
    stief_compress_append_joint_v,
    stief_compress_append_paged,
    stief_decode_attention,
    stief_decode_attention_q8,
    stief_append_decode_q8,
    stief_compress_append_q4,
    stief_compress_append_q8_paged,
    stief_decode_attention_q8_paged,
    stief_decode_attention_q4,
    stief_decode_attention_joint_v,
    stief_decode_attention_paged,
    stief_decode_attention_noalloc,
    stief_decode_auto_splits,
    stief_decode_latent,
    stief_decode_latent_joint_v,
    stief_decode_max_splits,
    stief_decode_workspace_bytes,
    stief_read_device_status,
    stief_status_string,
    workspace_for,
)
