"""Multi-pass EAGLE-3 TTT trunk+branch attention for NVIDIA B200 (sm_100a).

The computation lives in libttt_attn.so (C ABI, include/ttt_attn.h); this package
is its thin PyTorch binding.  Build the library with
``python -m attention_pass_rope_b200.build``.
"""

from .ops import (  # noqa: F401
    BlockLayout,
    Layout,
    block_attention,
    block_attn_bwd,
    block_attn_fwd,
    device_status,
    set_wait_budget_ns,
    ttt_attention,
    ttt_attn_bwd,
    ttt_attn_fwd,
    watchdog_selftest,
    workspace_bytes,
    workspace_layout,
)

__version__ = "0.3.0"
