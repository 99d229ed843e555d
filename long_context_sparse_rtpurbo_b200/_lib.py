"""ctypes loader of librtp.so and the C structs of include/rtp.h (argument marshalling only)."""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# RTP_LIBRARY_PATH selects another build of the same library (for example a tracing build)
LIB_PATH = os.environ.get("RTP_LIBRARY_PATH") or os.path.join(_HERE, "librtp.so")

RTP_OK, RTP_EINVAL, RTP_ESHAPE, RTP_EWORKSPACE, RTP_ECUDA, RTP_ETIMEOUT, RTP_EDEVICE, RTP_ECHECK = \
    0, -1, -2, -3, -4, -5, -6, -7

EXPORTS = (
    "rtp_status_str", "rtp_build_slot_map", "rtp_workspace_bytes", "rtp_workspace_init",
    "rtp_append_kv", "rtp_decode_step", "rtp_read_device_status", "rtp_last_launch_count",
    "rtp_decode_step_static", "rtp_decode_step_append", "rtp_decode_step_topk", "rtp_debug_set_wait_limit",
    "rtp_debug_fail_next_call", "rtp_prefill_workspace_bytes", "rtp_prefill",
)
RTP_STATIC_SCRATCH_BYTES = 16 << 20


class RtpLayerDesc(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32),
        ("head_dim", ctypes.c_int32), ("idx_dim", ctypes.c_int32),
        ("sinks", ctypes.c_int32), ("window", ctypes.c_int32), ("pad0", ctypes.c_int32),
        ("rope_base", ctypes.c_double), ("max_seq_len", ctypes.c_int64),
        ("slot_of_kv", ctypes.POINTER(ctypes.c_int32)),
    ]


class RtpCache(ctypes.Structure):
    _fields_ = [
        ("k_ret", ctypes.c_void_p), ("v_ret", ctypes.c_void_p), ("idx", ctypes.c_void_p),
        ("k_loc", ctypes.c_void_p), ("v_loc", ctypes.c_void_p),
        ("seq_off", ctypes.c_void_p), ("seq_cap", ctypes.c_void_p),
        ("T_total", ctypes.c_int64),
    ]


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load librtp.so; raises if it has not been built (there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"librtp.so not found at {path}; run __graft_entry__.build() first")
    lib = ctypes.CDLL(path)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    D, C = ctypes.POINTER(RtpLayerDesc), ctypes.POINTER(RtpCache)
    lib.rtp_status_str.restype = ctypes.c_char_p
    lib.rtp_status_str.argtypes = [ctypes.c_int]
    lib.rtp_build_slot_map.restype = ctypes.c_int
    lib.rtp_build_slot_map.argtypes = [vp, i32, vp, vp, vp]
    lib.rtp_workspace_bytes.restype = sz
    lib.rtp_workspace_bytes.argtypes = [D]
    lib.rtp_workspace_init.restype = ctypes.c_int
    lib.rtp_workspace_init.argtypes = [vp, sz, vp]
    lib.rtp_append_kv.restype = ctypes.c_int
    lib.rtp_append_kv.argtypes = [D, C, vp, vp, vp, vp, vp, i32, vp, vp]
    lib.rtp_decode_step.restype = ctypes.c_int
    lib.rtp_decode_step.argtypes = [D, C, vp, vp, vp, ctypes.c_double, vp, vp, vp, i64, vp, sz,
                                    vp]
    lib.rtp_decode_step_append.restype = ctypes.c_int
    lib.rtp_decode_step_append.argtypes = [D, C, vp, vp, vp, vp, vp, vp, ctypes.c_double, vp, vp,
                                           vp, i64, vp, sz, vp]
    lib.rtp_decode_step_topk.restype = ctypes.c_int
    lib.rtp_decode_step_topk.argtypes = [D, C, vp, vp, vp, i64, vp, vp, vp, i64, vp, sz, vp]
    lib.rtp_decode_step_static.restype = ctypes.c_int
    lib.rtp_decode_step_static.argtypes = [D, C, vp, vp, vp, ctypes.c_double, vp, vp, vp]
    lib.rtp_prefill_workspace_bytes.restype = sz
    lib.rtp_prefill_workspace_bytes.argtypes = [D, i32]
    lib.rtp_prefill.restype = ctypes.c_int
    lib.rtp_prefill.argtypes = [D, vp, vp, vp, vp, i32, vp, vp, sz, vp]
    lib.rtp_read_device_status.restype = ctypes.c_int
    lib.rtp_read_device_status.argtypes = [vp, vp]
    lib.rtp_last_launch_count.restype = i32
    lib.rtp_last_launch_count.argtypes = []
    lib.rtp_debug_set_wait_limit.restype = ctypes.c_int
    lib.rtp_debug_set_wait_limit.argtypes = [i64]
    lib.rtp_debug_fail_next_call.restype = ctypes.c_int
    lib.rtp_debug_fail_next_call.argtypes = [ctypes.c_int]
    _lib = lib
    return lib
