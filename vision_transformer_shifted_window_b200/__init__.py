"""B200-native shifted-window attention (Swin / SwinV2 / FlashSwin scores).

The computation lives in libswinattn.so (CUDA, sm_100a) behind the C ABI of
include/swin_attn.h; ``swin_attn`` is its thin ctypes binding.
"""
from .swin_attn import (  # noqa: F401
    SWIN_BF16, SWIN_F32, SWIN_MODE_COSINE_CPB, SWIN_MODE_DOT_BIAS, SWIN_MODE_ROPE, SwinError,
    swin_cpb_eval, swin_index_tables, swin_last_error, swin_stream_status, swin_version,
    swin_window_attn_fwd, swin_window_attn_workspace_size,
)
