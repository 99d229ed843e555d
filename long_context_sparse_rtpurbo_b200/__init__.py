"""RTPurbo per-layer sparse decode attention for B200 (sm_100a).

``rtp`` is the thin binding of librtp's C ABI (include/rtp.h); ``layer.DecodeLayer`` allocates
one layer's caches and workspace with PyTorch and drives the library.
"""
from . import rtp  # noqa: F401
from .rtp import (rtp_append_kv, rtp_build_slot_map, rtp_decode_step,  # noqa: F401
                  rtp_prefill, rtp_prefill_workspace_bytes, rtp_read_device_status, rtp_status_str, rtp_workspace_bytes, rtp_workspace_init)
