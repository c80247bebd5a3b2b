"""B200-native (sm_100a) decode hot path of Looped Latent Attention (LLA).

Source method: "Looped Latent Attention: Cross-Loop KV Compression for Looped
Transformers" (O'Neill & Reid, arXiv 2607.15456).

The compute lives in liblla.so (hand-written CUDA, C ABI in include/lla.h).
This package is its thin binding plus seeded synthetic inputs:

    from decode_attention_encode_b200 import lla_decode_attn, lla2d_decode_attn, lla_encode
"""

from ._lib import (  # noqa: F401
    EXPORTS,
    LLAError,
    device_status,
    kernel_timer,
    launch_timers,
    lib,
    library_path,
    lla2d_decode_attn,
    lla2d_decode_attn_paged,
    lla2d_decode_attn_paged_plan,
    lla2d_decode_attn_paged_planned,
    lla2d_decode_attn_paged_workspace,
    lla2d_decode_attn_rope,
    lla2d_decode_attn_workspace,
    lla_decode_attn,
    lla_decode_attn_noalloc,
    lla_decode_attn_paged,
    lla_decode_attn_paged_plan,
    lla_decode_attn_paged_planned,
    lla_decode_attn_paged_workspace,
    lla_decode_attn_rope,
    lla_decode_attn_workspace,
    lla_encode,
    lla_encode_bias,
    lla_encode_paged,
    lla_encode_with_bias,
    lla_encode_with_bias_workspace_bytes,
    lla_merge_attn,
)
